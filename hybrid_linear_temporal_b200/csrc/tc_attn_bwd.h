// tc_attn_bwd.h -- tensor-core (tcgen05) backward of the sliding-window
// attention branches for bf16, d_k = d_v = 128.
#pragma once
#include <cuda_runtime.h>

#include "hlta.h"
#include "kernels.h"

namespace hlta {

class TcAttnBwd {
public:
    // Returns nullptr when the configuration has no tensor-core path.
    static TcAttnBwd *create(const hlta_config &cfg);
    virtual ~TcAttnBwd() {}
    // True when run() takes this branch geometry over a full sequence of L tokens.
    virtual bool covers(int L, WindowGeom g) const = 0;
    // Gradients of one branch (gate_col 0 = SWA, 1 = DSWA), added to the fp32
    // accumulators dq, dk, dv [B, L, H, 128].  q, k are the tensors the forward
    // read; lse and rowdot [B, H, L] hold each query row's log2-domain
    // log-sum-exp and dout . o (the ungated branch output).
    virtual cudaError_t run(const void *q, const void *k, const void *v, const void *dout, int L, WindowGeom g,
                            const float *gates, int gate_col, const float *lse, const float *rowdot, float *dq,
                            float *dk, float *dv, int *dev_err, cudaStream_t s) = 0;
};

}  // namespace hlta
