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
// w_hi + 1, forward reach w - 1) and accumulates dk_j and dv_j.  A warp reads
// each row with one vector load (lane l holds d/32 consecutive elements) and
// reduces eight dot products at a time with shuffles.  fp32 math.
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

// Row access, warp-cooperative: lane l holds elements [l*E, l*E + E) of a row
// (E = d/32), read with one vector load, so a warp reads a whole row at once.
template <typename T, int E>
__device__ __forceinline__ void load_part(const T *row, int lane, float (&x)[E]) {
    if constexpr (sizeof(T) == 2) {
        if constexpr (E == 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(row + lane * 4);
            const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
            const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
            x[0] = __low2float(a);
            x[1] = __high2float(a);
            x[2] = __low2float(b);
            x[3] = __high2float(b);
        } else {
            const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(row + lane * 2);
            x[0] = __low2float(a);
            x[1] = __high2float(a);
        }
    } else {
        if constexpr (E == 4) {
            const float4 u = *reinterpret_cast<const float4 *>(row + lane * 4);
            x[0] = u.x;
            x[1] = u.y;
            x[2] = u.z;
            x[3] = u.w;
        } else {
            const float2 u = *reinterpret_cast<const float2 *>(row + lane * 2);
            x[0] = u.x;
            x[1] = u.y;
        }
    }
}

template <int E>
__device__ __forceinline__ float part_dot(const float (&a)[E], const float (&b)[E]) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) s = fmaf(a[e], b[e], s);
    return s;
}

// Reduces G independent per-lane partial sums across the warp (all lanes get
// every sum).
template <int G>
__device__ __forceinline__ void warp_sum_n(float (&x)[G]) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) x[g] += __shfl_xor_sync(0xffffffffu, x[g], o);
}

constexpr int kGrp = 8;  // keys (or queries) handled per group

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128) attn_bwd_q_kernel(AttnBwdArgs a) {
    constexpr int EK = DK / 32, EV = DV / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long row = (long long)blockIdx.x * 4 + wid;
    const long long total = (long long)a.B * a.L * a.H;
    if (row >= total) return;
    const int h = (int)(row % a.H);
    const long long i = (row / a.H) % a.L;
    const int b = (int)(row / ((long long)a.H * a.L));
    float q[EK], dO[EV];
    load_part<T, EK>(static_cast<const T *>(a.q) + (size_t)row * DK, lane, q);
    load_part<T, EV>(static_cast<const T *>(a.dout) + (size_t)row * DV, lane, dO);
#pragma unroll
    for (int e = 0; e < EK; ++e) q[e] *= a.scale_log2;

    const T *kb = static_cast<const T *>(a.k) + (size_t)b * a.L * a.H * DK;
    const T *vb = static_cast<const T *>(a.v) + (size_t)b * a.L * a.H * DV;
    auto krow = [&](long long p) { return kb + ((size_t)p * a.H + h) * DK; };
    auto vrow = [&](long long p) { return vb + ((size_t)p * a.H + h) * DV; };

    // pass 1: softmax statistics and the branch output o_i (online, log2 domain)
    float m_run = -INFINITY, l_run = 0.f, o[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) o[e] = 0.f;
    for_each_run(a.geom, i, a.L, [&](long long p0, int cnt) {
        for (int j0 = 0; j0 < cnt; j0 += kGrp) {
            float x[kGrp], vv[kGrp][EV];
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                float kk[EK];
                const long long p = p0 + min(j0 + g, cnt - 1);
                load_part<T, EK>(krow(p), lane, kk);
                load_part<T, EV>(vrow(p), lane, vv[g]);
                x[g] = part_dot<EK>(q, kk);
            }
            warp_sum_n<kGrp>(x);
            float mx = m_run;
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                if (j0 + g >= cnt) x[g] = -INFINITY;
                mx = fmaxf(mx, x[g]);
            }
            const float corr = exp2f(m_run - mx);
            l_run *= corr;
#pragma unroll
            for (int e = 0; e < EV; ++e) o[e] *= corr;
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                const float p = exp2f(x[g] - mx);
                l_run += p;
#pragma unroll
                for (int e = 0; e < EV; ++e) o[e] = fmaf(p, vv[g][e], o[e]);
            }
            m_run = mx;
        }
    });
    float rd[1] = {part_dot<EV>(o, dO)};
    warp_sum_n<1>(rd);
    const float rowdot = rd[0] / l_run;  // dout_i . o_i
    const float lse = m_run + log2f(l_run);
    if (lane == 0) {
        a.lse[row] = lse;
        a.rowdot[row] = rowdot;
    }
    const float gt = a.gates[h * 3 + a.gate_col];
    const float delta = gt * rowdot;

    // pass 2: dq_i = sum_j p_ij (g dout_i . v_j - delta_i) k_j / sqrt(d_k)
    float dq[EK];
#pragma unroll
    for (int e = 0; e < EK; ++e) dq[e] = 0.f;
    for_each_run(a.geom, i, a.L, [&](long long p0, int cnt) {
        for (int j0 = 0; j0 < cnt; j0 += kGrp) {
            float kk[kGrp][EK], sx[2 * kGrp];
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                float vv[EV];
                const long long p = p0 + min(j0 + g, cnt - 1);
                load_part<T, EK>(krow(p), lane, kk[g]);
                load_part<T, EV>(vrow(p), lane, vv);
                sx[g] = part_dot<EK>(q, kk[g]);
                sx[kGrp + g] = part_dot<EV>(dO, vv);
            }
            warp_sum_n<2 * kGrp>(sx);
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                const float ds = j0 + g < cnt ? exp2f(sx[g] - lse) * (gt * sx[kGrp + g] - delta) : 0.f;
#pragma unroll
                for (int e = 0; e < EK; ++e) dq[e] = fmaf(ds, kk[g][e], dq[e]);
            }
        }
    });
    float *dqp = a.dq + (size_t)row * DK + lane * EK;
#pragma unroll
    for (int e = 0; e < EK; ++e) dqp[e] += dq[e] * a.scale;
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128) attn_bwd_kv_kernel(AttnBwdArgs a) {
    constexpr int EK = DK / 32, EV = DV / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long row = (long long)blockIdx.x * 4 + wid;
    const long long total = (long long)a.B * a.L * a.H;
    if (row >= total) return;
    const int h = (int)(row % a.H);
    const long long j = (row / a.H) % a.L;
    const int b = (int)(row / ((long long)a.H * a.L));
    float k[EK], v[EV];
    load_part<T, EK>(static_cast<const T *>(a.k) + (size_t)row * DK, lane, k);
    load_part<T, EV>(static_cast<const T *>(a.v) + (size_t)row * DV, lane, v);
#pragma unroll
    for (int e = 0; e < EK; ++e) k[e] *= a.scale_log2;

    const size_t base_row = (size_t)b * a.L * a.H;
    const T *qb = static_cast<const T *>(a.q) + base_row * DK;
    const T *db = static_cast<const T *>(a.dout) + base_row * DV;
    const float gt = a.gates[h * 3 + a.gate_col];
    // queries whose window admits this key: r_k - w_hi <= r_q <= r_k + w - 1
    WindowGeom wt = a.geom;
    wt.w = a.geom.w_hi + 1;
    wt.w_hi = a.geom.w - 1;

    float dk[EK], dv[EV];
#pragma unroll
    for (int e = 0; e < EK; ++e) dk[e] = 0.f;
#pragma unroll
    for (int e = 0; e < EV; ++e) dv[e] = 0.f;
    for_each_run(wt, j, a.L, [&](long long p0, int cnt) {
        for (int j0 = 0; j0 < cnt; j0 += kGrp) {
            float qq[kGrp][EK], dd[kGrp][EV], sx[2 * kGrp];
            float lse[kGrp], rdt[kGrp];
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                const size_t qrow = (size_t)(p0 + min(j0 + g, cnt - 1)) * a.H + h;
                load_part<T, EK>(qb + qrow * DK, lane, qq[g]);
                load_part<T, EV>(db + qrow * DV, lane, dd[g]);
                lse[g] = a.lse[base_row + qrow];
                rdt[g] = a.rowdot[base_row + qrow];
                sx[g] = part_dot<EK>(qq[g], k);
                sx[kGrp + g] = part_dot<EV>(dd[g], v);
            }
            warp_sum_n<2 * kGrp>(sx);
#pragma unroll
            for (int g = 0; g < kGrp; ++g) {
                const bool act = j0 + g < cnt;
                const float p = act ? exp2f(sx[g] - lse[g]) : 0.f;
                const float ds = p * gt * (sx[kGrp + g] - rdt[g]);
                const float pg = p * gt;
#pragma unroll
                for (int e = 0; e < EK; ++e) dk[e] = fmaf(ds, qq[g][e], dk[e]);
#pragma unroll
                for (int e = 0; e < EV; ++e) dv[e] = fmaf(pg, dd[g][e], dv[e]);
            }
        }
    });
    float *dkp = a.dk + (size_t)row * DK + lane * EK;
    float *dvp = a.dv + (size_t)row * DV + lane * EV;
#pragma unroll
    for (int e = 0; e < EK; ++e) dkp[e] += dk[e] * a.scale;
#pragma unroll
    for (int e = 0; e < EV; ++e) dvp[e] += dv[e];
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
