// tc_gdn.h -- tensor-core chunked gated delta memory for bf16.
#pragma once
#include <cuda_runtime.h>

#include "hlta.h"

namespace hlta {

class TcGdn {
public:
    static TcGdn *create(const hlta_config &cfg, long long max_seq_len);
    virtual ~TcGdn() {}
    // True when run() would take a sequence of L tokens.
    virtual bool covers(int L) const = 0;
    virtual cudaError_t run(const void *q, const void *k, const void *v, const float *alpha,
                            const float *beta, int L, const float *S_in, float *S_out,
                            const float *gates, int mode, float *acc, void *out, int *dev_err,
                            cudaStream_t s, bool *done, int *launches) = 0;
};

}  // namespace hlta
