// tc_attention.h -- tensor-core (tcgen05) sliding-window attention for bf16.
#pragma once
#include <cuda_runtime.h>

#include "hlta.h"
#include "kernels.h"

namespace hlta {

// Scratch of the FP8 (e4m3) Q K^T path: q8, k8 [B, L, H, 128] bytes; sq, sk
// one scale per (segment, head, 128-row block), at least fp8_scale_floats()
// floats each.
struct Fp8Scratch {
    void *q8, *k8;
    float *sq, *sk;
};

// Scales one FP8 tensor needs at most, over both branch geometries.
size_t fp8_scale_floats(int B, int H, int max_len, int tokens_per_frame);

class TcAttention {
public:
    // Returns nullptr when the configuration has no tensor-core path.
    static TcAttention *create(const hlta_config &cfg, long long max_rows);
    virtual ~TcAttention() {}
    // One branch (gate_col 0 = SWA, 1 = DSWA) over a full sequence of L tokens.
    // Sets *done = false (and enqueues nothing) when this case is not covered,
    // so the caller runs the CUDA-core kernel instead.
    // acc2 (may be null) is a second fp32 accumulator added in the final modes.
    // lse_out (may be null) receives each row's log2-domain log-sum-exp, [B, H, L].
    // f8 (may be null): run Q K^T in e4m3 -- q and k are quantized first, with
    // one scale per 128-row tile of this branch's segments -- and P V in bf16.
    virtual cudaError_t run(const void *q, const void *k, const void *v, int L, WindowGeom g,
                            const float *gates, int gate_col, int mode, float *acc, const float *acc2,
                            void *out, int *dev_err, cudaStream_t s, bool *done,
                            float *lse_out = nullptr, const Fp8Scratch *f8 = nullptr) = 0;
    // True when run() would take this case (rather than leave it to the CUDA-core kernel).
    virtual bool covers(int L, WindowGeom g) const = 0;
};

}  // namespace hlta
