// bwd_util.cu -- the last steps of the layer backward: fp32 gradient
// accumulators to the tensor type (undoing the rotary embedding on the
// attention part of dq, dk), and the per-head gate gradients
// dgates[h, b] = sum over batch and tokens of dout . o_b.
#include "common.cuh"
#include "kernels.h"

namespace hlta {

namespace {

template <typename T>
__global__ void __launch_bounds__(256) bwd_finalize_kernel(BwdFinalizeArgs a) {
    const int half = a.d / 2;
    const long long pairs = a.rows * half;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < pairs;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long row = idx / half;
        const int m = (int)(idx % half);
        const size_t o = (size_t)row * a.d + 2 * m;
        float x0 = a.acc[o], x1 = a.acc[o + 1];
        if (a.att) {
            float g0 = a.att[o], g1 = a.att[o + 1];
            if (a.rope) {
                // transpose of the rotation by theta = t * inv_freq[m]
                const long long t = (row / a.H) % a.L;
                const double ang = fmod((double)t * a.inv_freq[m], 6.283185307179586476925286766559);
                float sn, cs;
                sincosf((float)ang, &sn, &cs);
                const float r0 = g0 * cs + g1 * sn, r1 = -g0 * sn + g1 * cs;
                g0 = r0;
                g1 = r1;
            }
            x0 += g0;
            x1 += g1;
        }
        T *out = static_cast<T *>(a.out);
        out[o] = from_f32<T>(x0);
        out[o + 1] = from_f32<T>(x1);
    }
}

__global__ void __launch_bounds__(256) gate_grad_kernel(const float *rowdot, int B, int L, int H, int col,
                                                        float *dgates) {
    const int h = blockIdx.x;
    float s = 0.f;
    for (long long i = threadIdx.x; i < (long long)B * L; i += blockDim.x) s += rowdot[i * H + h];
    s = warp_sum(s);
    __shared__ float part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += part[w];
        dgates[h * 3 + col] = t;
    }
}

// rowdot = dout . o per (b, t, h) row, in [B, L, H] and [B, H, L] order; one warp per row.
template <typename T>
__global__ void __launch_bounds__(256) rowdot_kernel(const T *dout, const float *o, long long rows, int d, int L,
                                                     int H, float *rowdot, float *rowdot_hm) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float s = 0.f;
    for (int c = lane; c < d; c += 32) s = fmaf(to_f32(dout[row * d + c]), o[row * d + c], s);
    s = warp_sum(s);
    if (lane == 0) {
        const int h = (int)(row % H);
        const long long t = (row / H) % L, b = row / ((long long)H * L);
        rowdot[row] = s;
        rowdot_hm[(b * H + h) * L + t] = s;
    }
}

}  // namespace

cudaError_t launch_rowdot(const void *dout, const float *o, long long rows, int d, int L, int H, bool bf16,
                          float *rowdot, float *rowdot_hm, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (bf16)
        rowdot_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(dout), o, rows, d, L,
                                                             H, rowdot, rowdot_hm);
    else
        rowdot_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float *>(dout), o, rows, d, L, H, rowdot,
                                                    rowdot_hm);
    return cudaGetLastError();
}

cudaError_t launch_bwd_finalize(const BwdFinalizeArgs &a, bool bf16, cudaStream_t s) {
    if (a.rows == 0) return cudaSuccess;
    if (a.d % 2 != 0 || a.d / 2 > 64) return cudaErrorInvalidValue;
    const long long pairs = a.rows * (a.d / 2);
    const unsigned blocks = (unsigned)(pairs < 148LL * 8 * 256 ? (pairs + 255) / 256 : 148 * 8);
    if (bf16)
        bwd_finalize_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a);
    else
        bwd_finalize_kernel<float><<<blocks, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gate_grad(const float *rowdot, int B, int L, int H, int col, float *dgates, cudaStream_t s) {
    gate_grad_kernel<<<H, 256, 0, s>>>(rowdot, B, L, H, col, dgates);
    return cudaGetLastError();
}

}  // namespace hlta
