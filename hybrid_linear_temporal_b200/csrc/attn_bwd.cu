// attn_bwd.cu -- CUDA-core backward pass of the SWA / DSWA branches.
//
// Kairos paper, section 2.2.2: the gradient of the softmax attention of Eq. (7)
// (SWA) and Eq. (8) (DSWA) with the window geometry of the forward kernels
// (backward reach w, forward reach w_hi, residue classes of frames).  For
// query i with admitted keys J(i), x_ij = q_i.k_j * log2(e)/sqrt(d_k),
// p_ij = 2^(x_ij - lse_i), and dO_i = g * dout_i (g the branch's gate):
//   delta_i = dO_i . o_i
//   dq_i = sum_j p_ij (dO_i.v_j - delta_i) k_j / sqrt(d_k)
//   dk_j = sum_i p_ij (dO_i.v_j - delta_i) q_i / sqrt(d_k)
//   dv_j = sum_i p_ij dO_i
// Two kernels: a query-major one (one warp per query row) that recomputes the
// row's softmax statistics and output, stores lse_i and dout_i.o_i, and
// accumulates dq_i; and a key-major one (one warp per key row) that walks the
// queries whose window admits the key (the transposed window: backward reach
// w_hi + 1, forward reach w - 1) and accumulates dk_j and dv_j.  fp32 math.
#include "common.cuh"
#include "kernels.h"

namespace hlta {

namespace {

// Calls f(p0, cnt) for runs of up to 32 consecutive token positions p0 .. p0+cnt-1
// that the window g admits for the token at position p (same residue class,
// rearranged position within [r - w + 1, r + w_hi], position below n_pos), from
// the latest class frame down.
template <typename F>
__device__ __forceinline__ void for_each_run(const WindowGeom &g, long long p, long long n_pos, F &&f) {
    const long long fr = p / g.P, s_i = p % g.P;
    const long long grp = fr % g.dil, m_i = fr / g.dil;
    const long long r = m_i * g.P + s_i;
    const long long r_lo = r - g.w + 1, r_hi = r + g.w_hi;
    const long long f_last = (n_pos - 1) / g.P;
    const long long m_last = f_last >= grp ? (f_last - grp) / g.dil : -1;
    const long long m_top = r_hi / g.P < m_last ? r_hi / g.P : m_last;
    for (long long m = m_top; m >= 0; --m) {
        const long long base_r = m * g.P;
        if (base_r + g.P - 1 < r_lo) break;
        const long long s_lo = r_lo - base_r > 0 ? r_lo - base_r : 0;
        const long long p_base = (grp + (long long)g.dil * m) * g.P;
        long long s_hi = (r_hi - base_r < g.P - 1) ? r_hi - base_r : g.P - 1;
        if (s_hi > n_pos - 1 - p_base) s_hi = n_pos - 1 - p_base;
        for (long long s0 = s_lo; s0 <= s_hi; s0 += 32)
            f(p_base + s0, (int)((s_hi - s0 + 1) < 32 ? (s_hi - s0 + 1) : 32));
    }
}

template <typename T, int DK>
__device__ __forceinline__ float dot_row(const T *x, const float *y) {
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < DK; ++c) acc = fmaf(to_f32(x[c]), y[c], acc);
    return acc;
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128) attn_bwd_q_kernel(AttnBwdArgs a) {
    constexpr int OK_ = DK / 32, OV = DV / 32;
    __shared__ float q_sh[4][DK];
    __shared__ float do_sh[4][DV];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long row = (long long)blockIdx.x * 4 + wid;
    const long long total = (long long)a.B * a.L * a.H;
    const bool live = row < total;
    const long long rr = live ? row : 0;
    const int h = (int)(rr % a.H);
    const long long i = (rr / a.H) % a.L;
    const int b = (int)(rr / ((long long)a.H * a.L));
    const T *qp = static_cast<const T *>(a.q) + (size_t)rr * DK;
    const T *dp_ = static_cast<const T *>(a.dout) + (size_t)rr * DV;
    for (int c = lane; c < DK; c += 32) q_sh[wid][c] = to_f32(qp[c]) * a.scale_log2;
    for (int c = lane; c < DV; c += 32) do_sh[wid][c] = to_f32(dp_[c]);
    __syncwarp();
    if (!live) return;

    const T *kb = static_cast<const T *>(a.k) + (size_t)b * a.L * a.H * DK;
    const T *vb = static_cast<const T *>(a.v) + (size_t)b * a.L * a.H * DV;
    auto krow = [&](long long p) { return kb + ((size_t)p * a.H + h) * DK; };
    auto vrow = [&](long long p) { return vb + ((size_t)p * a.H + h) * DV; };

    // pass 1: softmax statistics and the branch output o_i (online, log2 domain)
    float m_run = -INFINITY, l_run = 0.f, o[OV];
#pragma unroll
    for (int c = 0; c < OV; ++c) o[c] = 0.f;
    for_each_run(a.geom, i, a.L, [&](long long p0, int cnt) {
        const bool act = lane < cnt;
        const float x = act ? dot_row<T, DK>(krow(p0 + lane), q_sh[wid]) : -INFINITY;
        const float m_new = fmaxf(m_run, warp_max(x));
        const float corr = exp2f(m_run - m_new);
        const float pj = act ? exp2f(x - m_new) : 0.f;
        l_run = l_run * corr + warp_sum(pj);
#pragma unroll
        for (int c = 0; c < OV; ++c) o[c] *= corr;
        for (int j = 0; j < cnt; ++j) {
            const float pjj = __shfl_sync(0xffffffffu, pj, j);
            const T *vp = vrow(p0 + j);
#pragma unroll
            for (int c = 0; c < OV; ++c) o[c] = fmaf(pjj, to_f32(vp[lane + 32 * c]), o[c]);
        }
        m_run = m_new;
    });
    float part = 0.f;
#pragma unroll
    for (int c = 0; c < OV; ++c) part = fmaf(o[c], do_sh[wid][lane + 32 * c], part);
    const float rowdot = warp_sum(part) / l_run;  // dout_i . o_i
    const float lse = m_run + log2f(l_run);
    if (lane == 0) {
        a.lse[rr] = lse;
        a.rowdot[rr] = rowdot;
    }
    const float g = a.gates[h * 3 + a.gate_col];
    const float delta = g * rowdot;

    // pass 2: dq_i
    float dq[OK_];
#pragma unroll
    for (int c = 0; c < OK_; ++c) dq[c] = 0.f;
    for_each_run(a.geom, i, a.L, [&](long long p0, int cnt) {
        float ds = 0.f;
        if (lane < cnt) {
            const float x = dot_row<T, DK>(krow(p0 + lane), q_sh[wid]);
            const float p = exp2f(x - lse);
            const float dpv = g * dot_row<T, DV>(vrow(p0 + lane), do_sh[wid]);
            ds = p * (dpv - delta);
        }
        for (int j = 0; j < cnt; ++j) {
            const float dsj = __shfl_sync(0xffffffffu, ds, j);
            const T *kp = krow(p0 + j);
#pragma unroll
            for (int c = 0; c < OK_; ++c) dq[c] = fmaf(dsj, to_f32(kp[lane + 32 * c]), dq[c]);
        }
    });
    float *dqp = a.dq + (size_t)rr * DK;
#pragma unroll
    for (int c = 0; c < OK_; ++c) dqp[lane + 32 * c] += dq[c] * a.scale;
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128) attn_bwd_kv_kernel(AttnBwdArgs a) {
    constexpr int OK_ = DK / 32, OV = DV / 32;
    __shared__ float k_sh[4][DK];
    __shared__ float v_sh[4][DV];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long row = (long long)blockIdx.x * 4 + wid;
    const long long total = (long long)a.B * a.L * a.H;
    const bool live = row < total;
    const long long rr = live ? row : 0;
    const int h = (int)(rr % a.H);
    const long long j = (rr / a.H) % a.L;
    const int b = (int)(rr / ((long long)a.H * a.L));
    const T *kp = static_cast<const T *>(a.k) + (size_t)rr * DK;
    const T *vp = static_cast<const T *>(a.v) + (size_t)rr * DV;
    for (int c = lane; c < DK; c += 32) k_sh[wid][c] = to_f32(kp[c]) * a.scale_log2;
    for (int c = lane; c < DV; c += 32) v_sh[wid][c] = to_f32(vp[c]);
    __syncwarp();
    if (!live) return;

    const size_t base_row = (size_t)b * a.L * a.H;
    const T *qb = static_cast<const T *>(a.q) + base_row * DK;
    const T *db = static_cast<const T *>(a.dout) + base_row * DV;
    const float g = a.gates[h * 3 + a.gate_col];
    // queries whose window admits this key: r_k - w_hi <= r_q <= r_k + w - 1
    WindowGeom gt = a.geom;
    gt.w = a.geom.w_hi + 1;
    gt.w_hi = a.geom.w - 1;

    float dk[OK_], dv[OV];
#pragma unroll
    for (int c = 0; c < OK_; ++c) dk[c] = 0.f;
#pragma unroll
    for (int c = 0; c < OV; ++c) dv[c] = 0.f;
    for_each_run(gt, j, a.L, [&](long long p0, int cnt) {
        float p = 0.f, ds = 0.f;
        if (lane < cnt) {
            const long long qi = p0 + lane;
            const size_t qrow = (size_t)qi * a.H + h;
            const float x = dot_row<T, DK>(qb + qrow * DK, k_sh[wid]);
            p = exp2f(x - a.lse[base_row + qrow]);
            const float dpv = g * dot_row<T, DV>(db + qrow * DV, v_sh[wid]);
            ds = p * (dpv - g * a.rowdot[base_row + qrow]);
        }
        for (int jj = 0; jj < cnt; ++jj) {
            const float pg = g * __shfl_sync(0xffffffffu, p, jj);
            const float dsj = __shfl_sync(0xffffffffu, ds, jj);
            const size_t qrow = (size_t)(p0 + jj) * a.H + h;
            const T *qp = qb + qrow * DK;
            const T *dop = db + qrow * DV;
#pragma unroll
            for (int c = 0; c < OK_; ++c) dk[c] = fmaf(dsj, to_f32(qp[lane + 32 * c]), dk[c]);
#pragma unroll
            for (int c = 0; c < OV; ++c) dv[c] = fmaf(pg, to_f32(dop[lane + 32 * c]), dv[c]);
        }
    });
    float *dkp = a.dk + (size_t)rr * DK;
    float *dvp = a.dv + (size_t)rr * DV;
#pragma unroll
    for (int c = 0; c < OK_; ++c) dkp[lane + 32 * c] += dk[c] * a.scale;
#pragma unroll
    for (int c = 0; c < OV; ++c) dvp[lane + 32 * c] += dv[c];
}

template <typename T>
cudaError_t dispatch(const AttnBwdArgs &a, cudaStream_t s) {
    const long long total = (long long)a.B * a.L * a.H;
    const dim3 grid((unsigned)((total + 3) / 4));
#define HLTA_ATTN_BWD(DK, DV)                                  \
    if (a.d_k == DK && a.d_v == DV) {                          \
        attn_bwd_q_kernel<T, DK, DV><<<grid, 128, 0, s>>>(a);  \
        attn_bwd_kv_kernel<T, DK, DV><<<grid, 128, 0, s>>>(a); \
        return cudaGetLastError();                             \
    }
    HLTA_ATTN_BWD(128, 128)
    HLTA_ATTN_BWD(64, 64)
    HLTA_ATTN_BWD(128, 64)
    HLTA_ATTN_BWD(64, 128)
#undef HLTA_ATTN_BWD
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnBwdArgs &a, bool bf16, cudaStream_t s) {
    if ((long long)a.B * a.L * a.H == 0) return cudaSuccess;
    return bf16 ? dispatch<__nv_bfloat16>(a, s) : dispatch<float>(a, s);
}

}  // namespace hlta
