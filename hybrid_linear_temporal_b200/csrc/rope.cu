// rope.cu -- rotary position embedding of q and k for the attention branches.
//
// The pages name RoPE for the sliding-window blocks without fixing its form;
// the rotation used here is the reading stated in kernels.h: channel pair
// (2m, 2m+1) of the token at absolute position t is rotated by the angle
// t * base^(-2m/d).  The angle is formed and reduced modulo 2*pi in double
// precision, so the rotation stays exact to fp32 at long positions, and the
// result is rounded once to the tensor's element type.  One thread per pair of
// one (token, head); q and k are rotated by the same angles.
#include "common.cuh"
#include "kernels.h"

namespace hlta {

namespace {

template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(RopeArgs a) {
    const int half = a.d / 2;
    const long long total = (long long)a.B * a.n * a.H * half;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(idx % half);
        const long long row = idx / half;  // (b * n + t) * H + h
        const long long t = (row / a.H) % a.n;
        const double ang = fmod((double)(a.pos0 + t) * a.inv_freq[m], 6.283185307179586476925286766559);
        float sn, cs;
        sincosf((float)ang, &sn, &cs);
        const size_t off = (size_t)row * a.d + 2 * m;
        const T *q = static_cast<const T *>(a.q) + off;
        const T *k = static_cast<const T *>(a.k) + off;
        T *qo = static_cast<T *>(a.q_out) + off;
        T *ko = static_cast<T *>(a.k_out) + off;
        const float q0 = to_f32(q[0]), q1 = to_f32(q[1]), k0 = to_f32(k[0]), k1 = to_f32(k[1]);
        qo[0] = from_f32<T>(q0 * cs - q1 * sn);
        qo[1] = from_f32<T>(q0 * sn + q1 * cs);
        ko[0] = from_f32<T>(k0 * cs - k1 * sn);
        ko[1] = from_f32<T>(k0 * sn + k1 * cs);
    }
}

}  // namespace

cudaError_t launch_rope(const RopeArgs &a, bool bf16, cudaStream_t s) {
    if (a.d % 2 != 0 || a.d / 2 > 64) return cudaErrorInvalidValue;
    const long long total = (long long)a.B * a.n * a.H * (a.d / 2);
    if (total == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)(total < 148LL * 8 * 256 ? (total + 255) / 256 : 148 * 8);
    if (bf16)
        rope_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a);
    else
        rope_kernel<float><<<blocks, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace hlta
