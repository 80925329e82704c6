// attn_simt.cu -- CUDA-core softmax attention over the SWA / DSWA windows.
//
// Kairos paper, section 2.2.2: SWA (Eq. (7), causal window of w keys, or the
// centred window as printed) and DSWA (Eq. (8), SWA over residue classes of
// frames).  This kernel enumerates exactly the keys a query admits:
//   f = t / P, s = t % P, class g = f % dil, m = f / dil, r = m*P + s,
//   keys: frames f' = g + dil*m' and spatial s' with
//         r - w < m'*P + s' <= r + w_hi   (w_hi = 0: causal)
//   at positions below n_keys.
// SWA is the dil = 1 case.  fp32 arithmetic throughout; it serves the fp32
// configuration, sequences whose length is not a whole number of frames, and
// streaming steps.  The bf16 tensor-core kernel handles full sequences.
//
// One warp per query row; each lane scores one key of a group of 32, the warp
// keeps an online softmax (running max / sum in the log2 domain) and each lane
// accumulates d_v/32 output dimensions.
#include "common.cuh"
#include "kernels.h"

namespace hlta {

namespace {

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128) attn_simt_kernel(AttnSimtArgs a) {
    constexpr int OV = DV / 32;
    __shared__ float q_sh[4][DK];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long row = (long long)blockIdx.x * 4 + wid;
    const long long total = (long long)a.B * a.nq * a.H;
    const bool live = row < total;
    const long long rr = live ? row : 0;
    const int h = (int)(rr % a.H);
    const long long i = (rr / a.H) % a.nq;
    const int b = (int)(rr / ((long long)a.H * a.nq));

    const T *qp = static_cast<const T *>(a.q) + ((size_t)(b * (size_t)a.nq + i) * a.H + h) * DK;
    for (int c = lane; c < DK; c += 32) q_sh[wid][c] = to_f32(qp[c]) * a.scale_log2;
    __syncwarp();
    if (!live) return;

    const WindowGeom g = a.geom;
    const long long p_i = a.q_pos0 + i;
    const long long f_i = p_i / g.P, s_i = p_i % g.P;
    const long long grp = f_i % g.dil, m_i = f_i / g.dil;
    const long long r_i = m_i * g.P + s_i;
    const long long r_lo = r_i - g.w + 1, r_hi = r_i + g.w_hi;
    // the last class frame holding keys
    const long long f_last = (a.n_keys - 1) / g.P;
    const long long m_last = f_last >= grp ? (f_last - grp) / g.dil : -1;
    const long long m_top = r_hi / g.P < m_last ? r_hi / g.P : m_last;

    const T *kbase = static_cast<const T *>(a.k);
    const T *vbase = static_cast<const T *>(a.v);
    float m_run = -INFINITY, l_run = 0.f;
    float o[OV];
#pragma unroll
    for (int c = 0; c < OV; ++c) o[c] = 0.f;

    for (long long m = m_top; m >= 0; --m) {
        const long long base_r = m * g.P;
        if (base_r + g.P - 1 < r_lo) break;
        const long long s_lo = r_lo - base_r > 0 ? r_lo - base_r : 0;
        const long long p_base = (grp + (long long)g.dil * m) * g.P;
        long long s_hi = (r_hi - base_r < g.P - 1) ? r_hi - base_r : g.P - 1;
        if (s_hi > a.n_keys - 1 - p_base) s_hi = a.n_keys - 1 - p_base;
        for (long long s0 = s_lo; s0 <= s_hi; s0 += 32) {
            const long long s = s0 + lane;
            const bool act = s <= s_hi;
            float x = -INFINITY;
            if (act) {
                const long long kr = (p_base + s) % a.key_rows;
                const T *kp = kbase + ((size_t)(b * (size_t)a.key_rows + kr) * a.H + h) * DK;
                float acc = 0.f;
#pragma unroll 8
                for (int c = 0; c < DK; ++c) acc = fmaf(to_f32(kp[c]), q_sh[wid][c], acc);
                x = acc;
            }
            const float m_new = fmaxf(m_run, warp_max(x));
            const float corr = exp2f(m_run - m_new);
            const float pj = act ? exp2f(x - m_new) : 0.f;
            l_run = l_run * corr + warp_sum(pj);
#pragma unroll
            for (int c = 0; c < OV; ++c) o[c] *= corr;
            const int cnt = (int)((s_hi - s0 + 1) < 32 ? (s_hi - s0 + 1) : 32);
            for (int j = 0; j < cnt; ++j) {
                const float pjj = __shfl_sync(0xffffffffu, pj, j);
                const long long kr = (p_base + s0 + j) % a.key_rows;
                const T *vp = vbase + ((size_t)(b * (size_t)a.key_rows + kr) * a.H + h) * DV;
#pragma unroll
                for (int c = 0; c < OV; ++c) o[c] = fmaf(pjj, to_f32(vp[lane + 32 * c]), o[c]);
            }
            m_run = m_new;
        }
    }
    const float gate = a.gates[h * 3 + a.gate_col] / l_run;
    const size_t obase = ((size_t)(b * (size_t)a.nq + i) * a.H + h) * DV;
#pragma unroll
    for (int c = 0; c < OV; ++c)
        write_gated<T>(a.out_mode, a.acc, static_cast<T *>(a.out), obase + lane + 32 * c, gate * o[c]);
}

template <typename T>
cudaError_t dispatch(const AttnSimtArgs &a, cudaStream_t s) {
    const long long total = (long long)a.B * a.nq * a.H;
    const dim3 grid((unsigned)((total + 3) / 4));
    if (a.d_k == 128 && a.d_v == 128) attn_simt_kernel<T, 128, 128><<<grid, 128, 0, s>>>(a);
    else if (a.d_k == 64 && a.d_v == 64) attn_simt_kernel<T, 64, 64><<<grid, 128, 0, s>>>(a);
    else if (a.d_k == 128 && a.d_v == 64) attn_simt_kernel<T, 128, 64><<<grid, 128, 0, s>>>(a);
    else if (a.d_k == 64 && a.d_v == 128) attn_simt_kernel<T, 64, 128><<<grid, 128, 0, s>>>(a);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnSimtArgs &a, bool bf16, cudaStream_t s) {
    if ((long long)a.B * a.nq * a.H == 0) return cudaSuccess;
    return bf16 ? dispatch<__nv_bfloat16>(a, s) : dispatch<float>(a, s);
}

}  // namespace hlta
