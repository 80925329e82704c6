// gdn_recurrent.cu -- token-by-token gated delta memory (CUDA cores, fp32 state).
//
// Kairos paper, section 2.2.1 (Eq. (2)-(6), step 4):
//   v_old = alpha_t S_{t-1} k_t (decayed retrieval, the default form) or
//   v_old = S_{t-1} k_t (Eq. (2)/(6) as printed, HLTA_GDN_PAGES),
//   u_t = beta_t (v_t - v_old),  S_t = alpha_t S_{t-1} + u_t k_t^T,  o_t = S_t q_t.
// The rows of S (value dimension) evolve independently, so each warp owns a
// few rows across all d_k columns (d_k/32 columns per lane, vectorised loads)
// and the grid splits d_v across CTAs.  Per token the warp needs S k, S q and
// k.q (o_t = alpha_t (S_{t-1} q_t) + u_t (k_t . q_t)), all reduced in one
// interleaved butterfly round; the next token's inputs are prefetched while
// the current one is reduced.
//
// Used for the fp32 configuration, for streaming appends shorter than a chunk
// and as the tail of the chunked tensor-core path.
#include "common.cuh"
#include "kernels.h"

namespace hlta {

namespace {

constexpr int kWarps = 4;

template <typename T, int DK, int RPW>
struct TokenIn {
    float k[DK / 32], q[DK / 32], v[RPW], al, be;
};

template <typename T, int DK, int RPW>
__device__ __forceinline__ void load_token(TokenIn<T, DK, RPW> &x, const GdnRecArgs &a, size_t tok,
                                           int lane, int row0) {
    constexpr int CPL = DK / 32;
    const T *kp = static_cast<const T *>(a.k) + tok * DK + lane * CPL;
    const T *qp = static_cast<const T *>(a.q) + tok * DK + lane * CPL;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        x.k[j] = to_f32(kp[j]);
        x.q[j] = to_f32(qp[j]);
    }
    const T *vp = static_cast<const T *>(a.v) + tok * (size_t)a.d_v + row0;
#pragma unroll
    for (int r = 0; r < RPW; ++r) x.v[r] = to_f32(vp[r]);
    x.al = a.alpha[tok];
    x.be = a.beta[tok];
}

template <typename T, int DK, int RPW>
__global__ void __launch_bounds__(kWarps * 32) gdn_recurrent_kernel(GdnRecArgs a) {
    constexpr int CPL = DK / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh % a.H;
    const int row0 = (blockIdx.y * kWarps + warp) * RPW;
    if (row0 >= a.d_v) return;

    float S[RPW][CPL];
    const size_t sbase = ((size_t)bh * a.d_v + row0) * DK + lane * CPL;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int j = 0; j < CPL; ++j) S[r][j] = a.S_in ? a.S_in[sbase + (size_t)r * DK + j] : 0.f;

    const float gate = a.gates[h * 3 + 2];
    const bool printed = a.form == HLTA_GDN_PAGES;
    TokenIn<T, DK, RPW> cur, nxt;
    if (a.n > 0) load_token<T, DK, RPW>(cur, a, ((size_t)b * a.n) * a.H + h, lane, row0);
    for (int t = 0; t < a.n; ++t) {
        const size_t tok = ((size_t)b * a.n + t) * a.H + h;
        if (t + 1 < a.n) load_token<T, DK, RPW>(nxt, a, tok + a.H, lane, row0);
        float red[2 * RPW + 1];
        red[2 * RPW] = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) red[2 * RPW] = fmaf(cur.k[j], cur.q[j], red[2 * RPW]);
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                sk = fmaf(S[r][j], cur.k[j], sk);
                sq = fmaf(S[r][j], cur.q[j], sq);
            }
            red[2 * r] = sk;
            red[2 * r + 1] = sq;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int e = 0; e < 2 * RPW + 1; ++e) red[e] += __shfl_xor_sync(0xffffffffu, red[e], o);
        const float kq = red[2 * RPW];
        float outv = 0.f;
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const float u = cur.be * (cur.v[r] - (printed ? 1.f : cur.al) * red[2 * r]);
#pragma unroll
            for (int j = 0; j < CPL; ++j) S[r][j] = fmaf(cur.al, S[r][j], u * cur.k[j]);
            const float o_r = fmaf(cur.al, red[2 * r + 1], u * kq);
            if (lane == r) outv = o_r;
        }
        if (lane < RPW)
            write_gated<T>(a.out_mode, a.acc, static_cast<T *>(a.out), tok * a.d_v + row0 + lane,
                           gate * outv);
        cur = nxt;
    }
    if (a.S_out) {
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int j = 0; j < CPL; ++j) a.S_out[sbase + (size_t)r * DK + j] = S[r][j];
    }
}

template <typename T>
cudaError_t dispatch(const GdnRecArgs &a, cudaStream_t s) {
    constexpr int RPW = 4;
    if (a.d_v % (kWarps * RPW) != 0) return cudaErrorInvalidValue;
    const dim3 grid(a.B * a.H, a.d_v / (kWarps * RPW));
    if (a.d_k == 128) gdn_recurrent_kernel<T, 128, RPW><<<grid, kWarps * 32, 0, s>>>(a);
    else if (a.d_k == 64) gdn_recurrent_kernel<T, 64, RPW><<<grid, kWarps * 32, 0, s>>>(a);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gdn_recurrent(const GdnRecArgs &a, bool bf16, cudaStream_t s) {
    return bf16 ? dispatch<__nv_bfloat16>(a, s) : dispatch<float>(a, s);
}

// ---------------------------------------------------------------------------
// Streaming ring: keys/values of absolute position p live at row p % cap.
// ---------------------------------------------------------------------------
namespace {
__global__ void ring_append_kernel(RingAppendArgs a, int which) {
    const int d = which ? a.d_v : a.d_k;
    const size_t row_bytes = (size_t)a.H * d * a.elem_bytes;
    const size_t vec_per_row = row_bytes / 16;
    const size_t total = (size_t)a.B * a.n * vec_per_row;
    const uint4 *src = static_cast<const uint4 *>(which ? a.v : a.k);
    uint4 *dst = static_cast<uint4 *>(which ? a.ring_v : a.ring_k);
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
         idx += (size_t)gridDim.x * blockDim.x) {
        const size_t e = idx % vec_per_row;
        const size_t tok = idx / vec_per_row;  // b*n + t
        const size_t b = tok / a.n, t = tok % a.n;
        const size_t slot = (size_t)((a.pos0 + (long long)t) % a.cap);
        dst[(b * a.cap + slot) * vec_per_row + e] = src[idx];
    }
}
}  // namespace

cudaError_t launch_ring_append(const RingAppendArgs &a, cudaStream_t s) {
    for (int which = 0; which < 2; ++which) {
        const int d = which ? a.d_v : a.d_k;
        if (((size_t)a.H * d * a.elem_bytes) % 16 != 0) return cudaErrorInvalidValue;
        ring_append_kernel<<<296, 256, 0, s>>>(a, which);
    }
    return cudaGetLastError();
}

}  // namespace hlta
