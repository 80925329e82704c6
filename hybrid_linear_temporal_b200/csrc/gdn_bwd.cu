// gdn_bwd.cu -- backward pass of the gated delta memory, chunk form, on CUDA cores.
//
// Kairos paper, section 2.2.1: S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T)
// + beta_t v_t k_t^T, o_t = S_t q_t.  Inside a chunk of C = 64 tokens with
// start state S0, l_t = sum of log alpha up to t, gamma_t = e^{l_t}:
//   A_ts = beta_t e^{l_t - l_s} k_t.k_s (s < t),  T = (I + A)^-1
//   U    = T diag(beta) V - W S0^T,  W = T diag(beta gamma) K
//   O    = diag(gamma) Q S0^T + P U,  P_ts = e^{l_t - l_s} q_t.k_s (s <= t)
//   S_C  = gamma_C S0 + U^T diag(D) K,  D_s = e^{l_C - l_s}
// The backward (the chain rule through these, verified against the token
// recurrence's reverse mode) runs in four kernels:
//   gdn_bwd_prep   per chunk: T, W, T diag(beta) V, diag(D) K, and
//                  Lc = dO^T (diag(gamma) Q - P W)
//   gdn_bwd_fscan  per (b, h, 32 state rows), chunks in order: the chunk start
//                  states S0 and U (rows of S evolve independently)
//   gdn_bwd_dscan  per (b, h, 32 rows), chunks in reverse: the gradient of each
//                  chunk's end state, dS <- gamma_C dS - (dS (DK)^T) W + Lc
//   gdn_bwd_local  per chunk: dq, dk, dv, dalpha, dbeta and dout . o
// All arithmetic is fp32; matrix products use a shared-memory-tiled block GEMM.
#include "common.cuh"
#include "kernels.h"

namespace hlta {

namespace {

constexpr int kC = 64;        // chunk length
constexpr int kThreads = 256;
constexpr int kKT = 16;       // depth of one staged GEMM step

// A matrix operand: element (r, c) at p[r * rs + c * cs].
struct Mat {
    const float *p;
    long long rs, cs;
    __device__ float at(int r, int c) const { return p[r * rs + c * cs]; }
};
__device__ __forceinline__ Mat mat(const float *p, long long rs, long long cs) { return Mat{p, rs, cs}; }

// C(M x N) = alpha * A(M x K) B(K x N) + beta * C, for the whole block.
// A(m, k) = a.at(m, k), B(k, n) = b.at(k, n); rows >= m_valid of A read as zero
// and are not stored; beta == 0 does not read C.  stage: kKT * (M + N) floats of
// shared memory.  Thread (tm, tn) of a 16 x 16 grid owns rows tm + 16 i and
// columns tn + 16 j.  The operands of the next kKT-deep step are loaded into
// registers while the current step is computed.  Begins (before any operand is
// read) and ends with a block barrier.
template <int M, int N>
__device__ void block_gemm(Mat a, Mat b, int K, float *c, long long crs, long long ccs, float alpha, float beta,
                           float *stage, int m_valid = M) {
    constexpr int TM = M / 16, TN = N / 16;
    constexpr int LA = M * kKT / kThreads, LB = N * kKT / kThreads;  // staged elements per thread
    static_assert(LA * kThreads == M * kKT && LB * kThreads == N * kKT, "tile sizes");
    float *As = stage;            // [kKT][M]
    float *Bs = stage + kKT * M;  // [kKT][N]
    const int tid = threadIdx.x, tm = tid / 16, tn = tid % 16;
    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
    // staged element i of this thread: A (m, kk) and B (n, kk), laid out so that
    // consecutive threads read along the operand's contiguous direction
    auto a_idx = [&](int i, int &m, int &kk) {
        const int idx = tid + i * kThreads;
        if (a.cs == 1) { m = idx / kKT; kk = idx % kKT; } else { kk = idx / M; m = idx % M; }
    };
    auto b_idx = [&](int i, int &n, int &kk) {
        const int idx = tid + i * kThreads;
        if (b.cs == 1) { kk = idx / N; n = idx % N; } else { n = idx / kKT; kk = idx % kKT; }
    };
    float ra[LA], rb[LB];
    auto load = [&](int k0) {
#pragma unroll
        for (int i = 0; i < LA; ++i) {
            int m, kk;
            a_idx(i, m, kk);
            ra[i] = (k0 + kk < K && m < m_valid) ? a.at(m, k0 + kk) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < LB; ++i) {
            int n, kk;
            b_idx(i, n, kk);
            rb[i] = (k0 + kk < K) ? b.at(k0 + kk, n) : 0.f;
        }
    };
    // the operands may have been written by other threads just before the call
    __syncthreads();
    load(0);
    for (int k0 = 0; k0 < K; k0 += kKT) {
        if (k0 > 0) __syncthreads();  // every thread has finished reading the stage
#pragma unroll
        for (int i = 0; i < LA; ++i) {
            int m, kk;
            a_idx(i, m, kk);
            As[kk * M + m] = ra[i];
        }
#pragma unroll
        for (int i = 0; i < LB; ++i) {
            int n, kk;
            b_idx(i, n, kk);
            Bs[kk * N + n] = rb[i];
        }
        __syncthreads();
        if (k0 + kKT < K) load(k0 + kKT);
#pragma unroll 4
        for (int kk = 0; kk < kKT; ++kk) {
            float av[TM], bv[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) av[i] = As[kk * M + tm + 16 * i];
#pragma unroll
            for (int j = 0; j < TN; ++j) bv[j] = Bs[kk * N + tn + 16 * j];
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int m = tm + 16 * i;
        if (m >= m_valid) continue;
#pragma unroll
        for (int j = 0; j < TN; ++j) {
            float *cp = c + m * crs + (tn + 16 * j) * ccs;
            *cp = beta == 0.f ? alpha * acc[i][j] : fmaf(beta, *cp, alpha * acc[i][j]);
        }
    }
    __syncthreads();
}

struct ChunkScalars {
    float ell[kC], gam[kC], D[kC], be[kC], al[kC];
};

// Loads the chunk's scalars: l_t (log alpha summed from the chunk start), gamma,
// D_t = e^{l_last - l_t}, beta; padded tokens (t >= n) are identity steps
// (alpha = 1, beta = 0).
__device__ void load_scalars(ChunkScalars &sc, const GdnBwdArgs &a, int b, int h, int t0, int n) {
    const int tid = threadIdx.x;
    if (tid < kC) {
        const size_t row = ((size_t)b * a.L + t0 + tid) * a.H + h;
        sc.al[tid] = tid < n ? a.alpha[row] : 1.f;
        sc.be[tid] = tid < n ? a.beta[row] : 0.f;
        sc.ell[tid] = logf(sc.al[tid]);
    }
    __syncthreads();
    if (tid < 32) {  // inclusive prefix sum over 64 entries, two per lane
        float x0 = sc.ell[2 * tid], x1 = sc.ell[2 * tid + 1];
        float s = x0 + x1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, o);
            if (tid >= o) s += y;
        }
        sc.ell[2 * tid] = s - x1;
        sc.ell[2 * tid + 1] = s;
    }
    __syncthreads();
    if (tid < kC) {
        sc.gam[tid] = expf(sc.ell[tid]);
        sc.D[tid] = expf(sc.ell[kC - 1] - sc.ell[tid]);
    }
    __syncthreads();
}

// dst[t][c] = scale * src row (b, t0 + t, h) for t < n, zero for padded rows.
template <typename T>
__device__ void load_rows(float *dst, const void *src, int d, const GdnBwdArgs &a, int b, int h, int t0, int n) {
    const T *s = static_cast<const T *>(src);
    for (int idx = threadIdx.x; idx < kC * d; idx += kThreads) {
        const int t = idx / d, c = idx % d;
        dst[idx] = t < n ? to_f32(s[(((size_t)b * a.L + t0 + t) * a.H + h) * d + c]) : 0.f;
    }
}

// ---------------------------------------------------------------------------
// gdn_bwd_prep: one chunk per iteration of a persistent CTA.
// ---------------------------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kThreads) gdn_bwd_prep(GdnBwdArgs a) {
    __shared__ ChunkScalars sc;
    __shared__ float Tm[kC][kC + 1];
    __shared__ float stage[kKT * (DK > DV ? 2 * DK : 2 * DV)];
    float *ws = a.ws + (size_t)blockIdx.x * a.ws_per_cta;
    float *Qc = ws, *Kc = Qc + kC * DK, *Vc = Kc + kC * DK, *dOc = Vc + kC * DV;
    float *KK = dOc + kC * DV, *P = KK + kC * kC, *Y = P + kC * kC, *Kb = Y + kC * DK, *Vb = Kb + kC * DK;
    const int nc = (a.L + kC - 1) / kC;
    const int tid = threadIdx.x;
    for (long long it = blockIdx.x; it < (long long)a.B * a.H * nc; it += gridDim.x) {
        const int bh = (int)(it / nc), ci = (int)(it % nc);
        const int b = bh / a.H, h = bh % a.H, t0 = ci * kC, n = min(kC, a.L - t0);
        const size_t cidx = (size_t)bh * nc + ci;
        load_scalars(sc, a, b, h, t0, n);
        load_rows<T>(Qc, a.q, DK, a, b, h, t0, n);
        load_rows<T>(Kc, a.k, DK, a, b, h, t0, n);
        load_rows<T>(Vc, a.v, DV, a, b, h, t0, n);
        load_rows<T>(dOc, a.dout, DV, a, b, h, t0, n);
        __syncthreads();
        // K K^T and Q K^T
        block_gemm<kC, kC>(mat(Kc, DK, 1), mat(Kc, 1, DK), DK, KK, kC, 1, 1.f, 0.f, stage);
        block_gemm<kC, kC>(mat(Qc, DK, 1), mat(Kc, 1, DK), DK, P, kC, 1, 1.f, 0.f, stage);
        // A (strictly lower) into Tm; P masked with the decay ratios
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            const int t = idx / kC, s = idx % kC;
            const float e = s <= t ? expf(sc.ell[t] - sc.ell[s]) : 0.f;
            Tm[t][s] = s < t ? sc.be[t] * e * KK[idx] : 0.f;
            P[idx] = e * P[idx];
        }
        __syncthreads();
        // T = (I + A)^-1 by forward substitution, one column per thread, written
        // straight to the chunk's T in global memory
        float *Tg = a.bw_T + cidx * kC * kC;
        if (tid < kC) {
            const int j = tid;
            float x[kC];
#pragma unroll
            for (int t = 0; t < kC; ++t) {
                float s = t == j ? 1.f : 0.f;
                for (int r = j; r < t; ++r) s = fmaf(-Tm[t][r], x[r], s);
                x[t] = t < j ? 0.f : s;
                Tg[t * kC + j] = x[t];
            }
        }
        // scaled operands: Kb = diag(beta gamma) K, Vb = diag(beta) V, Kd = diag(D) K
        float *Kd = a.bw_Kd + cidx * kC * DK;
        for (int idx = tid; idx < kC * DK; idx += kThreads) {
            const int t = idx / DK;
            Kb[idx] = sc.be[t] * sc.gam[t] * Kc[idx];
            Kd[idx] = sc.D[t] * Kc[idx];
            Y[idx] = sc.gam[t] * Qc[idx];
        }
        for (int idx = tid; idx < kC * DV; idx += kThreads) Vb[idx] = sc.be[idx / DV] * Vc[idx];
        if (tid < kC) a.bw_ell[cidx * kC + tid] = sc.ell[tid];
        __syncthreads();
        float *W = a.bw_W + cidx * kC * DK;
        float *TbV = a.bw_TbV + cidx * kC * DV;
        block_gemm<kC, DK>(mat(Tg, kC, 1), mat(Kb, DK, 1), kC, W, DK, 1, 1.f, 0.f, stage);
        block_gemm<kC, DV>(mat(Tg, kC, 1), mat(Vb, DV, 1), kC, TbV, DV, 1, 1.f, 0.f, stage);
        // Y = diag(gamma) Q - P W;  Lc = g dO^T Y
        block_gemm<kC, DK>(mat(P, kC, 1), mat(W, DK, 1), kC, Y, DK, 1, -1.f, 1.f, stage);
        const float g = a.gates[h * 3 + 2];
        block_gemm<DV, DK>(mat(dOc, 1, DV), mat(Y, DK, 1), kC, a.bw_Lc + cidx * DV * DK, DK, 1, g, 0.f, stage);
    }
}

// Asynchronous 16-byte global -> shared copies (completion by commit groups).
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// n floats (a multiple of 4, 16-byte aligned at both ends) by the whole block
__device__ __forceinline__ void copy_async(float *dst, const float *src, int n) {
    for (int i = threadIdx.x * 4; i < n; i += kThreads * 4) cp_async16(dst + i, src + i);
}

constexpr int kScanRows = 32;  // state rows per scan CTA

template <int DK, int DV>
constexpr size_t fscan_smem_floats() {
    return 2 * (2 * (size_t)kC * DK + (size_t)kC * kScanRows + 4) + (size_t)kScanRows * DK + kC * kScanRows +
           kKT * (kScanRows + DK);
}
template <int DK, int DV>
constexpr size_t dscan_smem_floats() {
    return 2 * (2 * (size_t)kC * DK + (size_t)kScanRows * DK + 4) + (size_t)kScanRows * DK + kScanRows * kC +
           kKT * (kScanRows + DK);
}

// ---------------------------------------------------------------------------
// gdn_bwd_fscan: chunk start states and U, 32 rows of S per CTA.  The next
// chunk's W, diag(D) K, the row slice of T diag(beta) V and l_C are copied into
// shared memory (double buffer) while the current chunk is computed.
// ---------------------------------------------------------------------------
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) gdn_bwd_fscan(GdnBwdArgs a) {
    constexpr int R = kScanRows;
    extern __shared__ __align__(16) float fsm[];
    float *buf[2];
    buf[0] = fsm;
    buf[1] = fsm + (2 * kC * DK + kC * R + 4);
    float *Sr = fsm + 2 * (2 * kC * DK + kC * R + 4);
    float *Ub = Sr + R * DK;
    float *stage = Ub + kC * R;
    const int r0 = blockIdx.x * R, bh = blockIdx.y;
    const int nc = (a.L + kC - 1) / kC;
    const int tid = threadIdx.x;
    // buffer layout: W [kC][DK], Kd [kC][DK], TbV rows slice [kC][R], l (4 floats, the last is l_C)
    auto prefetch = [&](int ci, float *bf) {
        const size_t cidx = (size_t)bh * nc + ci;
        copy_async(bf, a.bw_W + cidx * kC * DK, kC * DK);
        copy_async(bf + kC * DK, a.bw_Kd + cidx * kC * DK, kC * DK);
        const float *TbV = a.bw_TbV + cidx * kC * DV + r0;
        for (int i = tid; i < kC * (R / 4); i += kThreads)
            cp_async16(bf + 2 * kC * DK + (i / (R / 4)) * R + (i % (R / 4)) * 4, TbV + (i / (R / 4)) * DV + (i % (R / 4)) * 4);
        if (tid == 0) cp_async16(bf + 2 * kC * DK + kC * R, a.bw_ell + cidx * kC + kC - 4);
    };
    for (int idx = tid; idx < R * DK; idx += kThreads)
        Sr[idx] = a.S0 ? a.S0[((size_t)bh * DV + r0 + idx / DK) * DK + idx % DK] : 0.f;
    prefetch(0, buf[0]);
    cp_async_commit();
    for (int ci = 0; ci < nc; ++ci) {
        if (ci + 1 < nc) prefetch(ci + 1, buf[(ci + 1) & 1]);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();
        const float *bf = buf[ci & 1];
        const size_t cidx = (size_t)bh * nc + ci;
        float *Sg = a.bw_S + cidx * DV * DK + (size_t)r0 * DK;
        for (int idx = tid; idx < R * DK; idx += kThreads) Sg[idx] = Sr[idx];
        // U[:, rows] = T diag(beta) V[:, rows] - W S_rows^T
        for (int idx = tid; idx < kC * R; idx += kThreads) Ub[idx] = bf[2 * kC * DK + idx];
        block_gemm<kC, R>(mat(bf, DK, 1), mat(Sr, 1, DK), DK, Ub, R, 1, -1.f, 1.f, stage);
        float *Ug = a.bw_U + cidx * kC * DV;
        for (int idx = tid; idx < kC * R; idx += kThreads) Ug[(idx / R) * DV + r0 + idx % R] = Ub[idx];
        // S_rows <- gamma_C S_rows + U[:, rows]^T diag(D) K
        const float gC = expf(bf[2 * kC * DK + kC * R + 3]);
        block_gemm<R, DK>(mat(Ub, 1, R), mat(bf + kC * DK, DK, 1), kC, Sr, DK, 1, 1.f, gC, stage);
    }
}

// ---------------------------------------------------------------------------
// gdn_bwd_dscan: gradients of the chunk end states, chunks in reverse, with the
// same double-buffered prefetch (diag(D) K, W, the rows of Lc, l_C).
// ---------------------------------------------------------------------------
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) gdn_bwd_dscan(GdnBwdArgs a) {
    constexpr int R = kScanRows;
    extern __shared__ __align__(16) float dsm[];
    float *buf[2];
    buf[0] = dsm;
    buf[1] = dsm + (2 * kC * DK + R * DK + 4);
    float *dS = dsm + 2 * (2 * kC * DK + R * DK + 4);
    float *X = dS + R * DK;
    float *stage = X + R * kC;
    const int r0 = blockIdx.x * R, bh = blockIdx.y;
    const int nc = (a.L + kC - 1) / kC;
    const int tid = threadIdx.x;
    // buffer layout: W [kC][DK], Kd [kC][DK], Lc rows [R][DK], l (4 floats)
    auto prefetch = [&](int ci, float *bf) {
        const size_t cidx = (size_t)bh * nc + ci;
        copy_async(bf, a.bw_W + cidx * kC * DK, kC * DK);
        copy_async(bf + kC * DK, a.bw_Kd + cidx * kC * DK, kC * DK);
        copy_async(bf + 2 * kC * DK, a.bw_Lc + cidx * DV * DK + (size_t)r0 * DK, R * DK);
        if (tid == 0) cp_async16(bf + 2 * kC * DK + R * DK, a.bw_ell + cidx * kC + kC - 4);
    };
    for (int idx = tid; idx < R * DK; idx += kThreads)
        dS[idx] = a.dS_final ? a.dS_final[((size_t)bh * DV + r0 + idx / DK) * DK + idx % DK] : 0.f;
    prefetch(nc - 1, buf[(nc - 1) & 1]);
    cp_async_commit();
    for (int ci = nc - 1; ci >= 0; --ci) {
        if (ci > 0) prefetch(ci - 1, buf[(ci - 1) & 1]);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();
        const float *bf = buf[ci & 1];
        const size_t cidx = (size_t)bh * nc + ci;
        float *dSg = a.bw_dS + cidx * DV * DK + (size_t)r0 * DK;
        for (int idx = tid; idx < R * DK; idx += kThreads) dSg[idx] = dS[idx];
        // X = dS_rows (diag(D) K)^T
        block_gemm<R, kC>(mat(dS, DK, 1), mat(bf + kC * DK, 1, DK), DK, X, kC, 1, 1.f, 0.f, stage);
        // dS_rows <- gamma_C dS_rows - X W + Lc[rows]
        const float gC = expf(bf[2 * kC * DK + R * DK + 3]);
        block_gemm<R, DK>(mat(X, kC, 1), mat(bf, DK, 1), kC, dS, DK, 1, -1.f, gC, stage);
        for (int idx = tid; idx < R * DK; idx += kThreads) dS[idx] += bf[2 * kC * DK + idx];
        __syncthreads();
    }
    if (a.dS0)
        for (int idx = tid; idx < R * DK; idx += kThreads)
            a.dS0[((size_t)bh * DV + r0 + idx / DK) * DK + idx % DK] = dS[idx];
}

// ---------------------------------------------------------------------------
// gdn_bwd_local: the token gradients of one chunk per iteration.
// ---------------------------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2) gdn_bwd_local(GdnBwdArgs a) {
    __shared__ ChunkScalars sc;
    __shared__ float dl[kC];
    __shared__ float red[kC][4];
    __shared__ float stage[kKT * (DK > DV ? 2 * DK : 2 * DV)];
    float *ws = a.ws + (size_t)blockIdx.x * a.ws_per_cta;
    float *Qc = ws, *Kc = Qc + kC * DK, *Vc = Kc + kC * DK, *dOc = Vc + kC * DV;
    float *KK = dOc + kC * DV, *P = KK + kC * kC, *dA = P + kC * kC, *MdOU = dA + kC * kC, *Es = MdOU + kC * kC;
    float *QS = Es + kC * kC, *KS = QS + kC * DV, *KdS = KS + kC * DV, *dU = KdS + kC * DV, *dR = dU + kC * DV;
    float *Gq = dR + kC * DV, *Gk = Gq + kC * DK, *tmp = Gk + kC * DK;
    const int nc = (a.L + kC - 1) / kC;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (long long it = blockIdx.x; it < (long long)a.B * a.H * nc; it += gridDim.x) {
        const int bh = (int)(it / nc), ci = (int)(it % nc);
        const int b = bh / a.H, h = bh % a.H, t0 = ci * kC, n = min(kC, a.L - t0);
        const size_t cidx = (size_t)bh * nc + ci;
        const float g = a.gates[h * 3 + 2];
        load_scalars(sc, a, b, h, t0, n);
        load_rows<T>(Qc, a.q, DK, a, b, h, t0, n);
        load_rows<T>(Kc, a.k, DK, a, b, h, t0, n);
        load_rows<T>(Vc, a.v, DV, a, b, h, t0, n);
        load_rows<T>(dOc, a.dout, DV, a, b, h, t0, n);
        const float *S0 = a.bw_S + cidx * DV * DK, *dSC = a.bw_dS + cidx * DV * DK;
        const float *U = a.bw_U + cidx * kC * DV, *Tg = a.bw_T + cidx * kC * kC;
        __syncthreads();
        block_gemm<kC, kC>(mat(Kc, DK, 1), mat(Kc, 1, DK), DK, KK, kC, 1, 1.f, 0.f, stage);
        block_gemm<kC, kC>(mat(Qc, DK, 1), mat(Kc, 1, DK), DK, P, kC, 1, 1.f, 0.f, stage);
        block_gemm<kC, DV>(mat(Qc, DK, 1), mat(S0, 1, DK), DK, QS, DV, 1, 1.f, 0.f, stage);
        block_gemm<kC, DV>(mat(Kc, DK, 1), mat(S0, 1, DK), DK, KS, DV, 1, 1.f, 0.f, stage);
        block_gemm<kC, DV>(mat(Kc, DK, 1), mat(dSC, 1, DK), DK, KdS, DV, 1, 1.f, 0.f, stage);
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            const int t = idx / kC, s = idx % kC;
            P[idx] = s <= t ? expf(sc.ell[t] - sc.ell[s]) * P[idx] : 0.f;
        }
        // O = diag(gamma) Q S0^T + P U (into tmp), for dout . o
        for (int idx = tid; idx < kC * DV; idx += kThreads) tmp[idx] = sc.gam[idx / DV] * QS[idx];
        block_gemm<kC, DV>(mat(P, kC, 1), mat(U, DV, 1), kC, tmp, DV, 1, 1.f, 1.f, stage);
        for (int t = warp; t < n; t += kThreads / 32) {
            float s = 0.f;
            for (int c = lane; c < DV; c += 32) s = fmaf(dOc[t * DV + c], tmp[t * DV + c], s);
            s = warp_sum(s);
            if (lane == 0) a.rowdot[((size_t)b * a.L + t0 + t) * a.H + h] = s;
        }
        // dU = diag(D) K dS_C^T + g P^T dO;  dR = T^T dU
        for (int idx = tid; idx < kC * DV; idx += kThreads) dU[idx] = sc.D[idx / DV] * KdS[idx];
        block_gemm<kC, DV>(mat(P, 1, kC), mat(dOc, DV, 1), kC, dU, DV, 1, g, 1.f, stage);
        block_gemm<kC, DV>(mat(Tg, 1, kC), mat(dU, DV, 1), kC, dR, DV, 1, 1.f, 0.f, stage);
        // dA = -dR U^T (strictly lower), dOU = g dO U^T
        block_gemm<kC, kC>(mat(dR, DV, 1), mat(U, 1, DV), DV, dA, kC, 1, -1.f, 0.f, stage);
        block_gemm<kC, kC>(mat(dOc, DV, 1), mat(U, 1, DV), DV, MdOU, kC, 1, g, 0.f, stage);
        // dl: per-token derivative of l_t (accumulated below in pieces)
        if (tid < kC) dl[tid] = 0.f;
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            const int t = idx / kC, s = idx % kC;
            const float e = s <= t ? expf(sc.ell[t] - sc.ell[s]) : 0.f;
            if (s >= t) dA[idx] = 0.f;
            // Es = E + E^T, E_ts = dA_ts beta_t e_ts (s < t); written from both sides
            const float dM = MdOU[idx] * P[idx];        // d l through P: +row t, -column s
            const float Am = s < t ? dA[idx] * sc.be[t] * e * KK[idx] : 0.f;  // through A
            MdOU[idx] *= e;
            tmp[idx] = dM + Am;                          // row/column sums below
            (void)0;
        }
        __syncthreads();
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            const int t = idx / kC, s = idx % kC;
            const float ets = s < t ? expf(sc.ell[t] - sc.ell[s]) : 0.f;
            const float est = t < s ? expf(sc.ell[s] - sc.ell[t]) : 0.f;
            Es[idx] = (s < t ? dA[idx] * sc.be[t] * ets : 0.f) + (t < s ? dA[s * kC + t] * sc.be[s] * est : 0.f);
        }
        __syncthreads();
        // dl_t += sum_s (dM + Am)_ts - sum_s (dM + Am)_st
        if (tid < kC) {
            float rs = 0.f, cs = 0.f;
            for (int s = 0; s < kC; ++s) {
                rs += tmp[tid * kC + s];
                cs += tmp[s * kC + tid];
            }
            dl[tid] += rs - cs;
        }
        __syncthreads();
        // dQ = g diag(gamma) dO S0 + (M . dOU) K
        block_gemm<kC, DK>(mat(dOc, DV, 1), mat(S0, DK, 1), DV, Gq, DK, 1, 1.f, 0.f, stage);
        for (int idx = tid; idx < kC * DK; idx += kThreads) Gq[idx] *= g * sc.gam[idx / DK];
        block_gemm<kC, DK>(mat(MdOU, kC, 1), mat(Kc, DK, 1), kC, Gq, DK, 1, 1.f, 1.f, stage);
        // dK = diag(D) U dS_C - diag(beta gamma) dR S0 + (M . dOU)^T Q + Es K
        block_gemm<kC, DK>(mat(U, DV, 1), mat(dSC, DK, 1), DV, Gk, DK, 1, 1.f, 0.f, stage);
        block_gemm<kC, DK>(mat(dR, DV, 1), mat(S0, DK, 1), DV, tmp, DK, 1, 1.f, 0.f, stage);
        for (int idx = tid; idx < kC * DK; idx += kThreads) {
            const int t = idx / DK;
            Gk[idx] = sc.D[t] * Gk[idx] - sc.be[t] * sc.gam[t] * tmp[idx];
        }
        block_gemm<kC, DK>(mat(MdOU, 1, kC), mat(Qc, DK, 1), kC, Gk, DK, 1, 1.f, 1.f, stage);
        block_gemm<kC, DK>(mat(Es, kC, 1), mat(Kc, DK, 1), kC, Gk, DK, 1, 1.f, 1.f, stage);
        // per-token reductions: warp w handles tokens w, w + 8, ...
        for (int t = warp; t < kC; t += kThreads / 32) {
            float r_dv = 0.f, r_ks = 0.f, r_qs = 0.f, r_d = 0.f;
            for (int c = lane; c < DV; c += 32) {
                r_dv = fmaf(dR[t * DV + c], Vc[t * DV + c], r_dv);
                r_ks = fmaf(dR[t * DV + c], KS[t * DV + c], r_ks);
                r_qs = fmaf(dOc[t * DV + c], QS[t * DV + c], r_qs);
                r_d = fmaf(U[t * DV + c], KdS[t * DV + c], r_d);
            }
            float r_a = 0.f;
            for (int s = lane; s < t; s += 32) r_a = fmaf(dA[t * kC + s], expf(sc.ell[t] - sc.ell[s]) * KK[t * kC + s], r_a);
            r_dv = warp_sum(r_dv);
            r_ks = warp_sum(r_ks);
            r_qs = warp_sum(r_qs);
            r_d = warp_sum(r_d);
            r_a = warp_sum(r_a);
            if (lane == 0) {
                red[t][0] = r_dv - sc.gam[t] * r_ks + r_a;  // dbeta_t
                red[t][1] = sc.D[t] * r_d;                    // dD_t * D_t
                dl[t] += g * sc.gam[t] * r_qs - sc.gam[t] * sc.be[t] * r_ks - sc.D[t] * r_d;
            }
        }
        // <dS_C, S0> for the gamma_C term
        float part = 0.f;
        for (int idx = tid; idx < DV * DK; idx += kThreads) part = fmaf(dSC[idx], S0[idx], part);
        part = warp_sum(part);
        if (lane == 0) red[warp][2] = part;
        __syncthreads();
        if (tid == 0) {
            float sd = 0.f, ip = 0.f;
            for (int t = 0; t < kC; ++t) sd += red[t][1];
            for (int w = 0; w < kThreads / 32; ++w) ip += red[w][2];
            dl[kC - 1] += sd + sc.gam[kC - 1] * ip;
            // d log alpha_tau = sum_{t >= tau} dl_t
            float acc = 0.f;
            for (int t = kC - 1; t >= 0; --t) {
                acc += dl[t];
                red[t][3] = acc;
            }
        }
        __syncthreads();
        // write the token gradients (the memory branch stores; attention adds)
        for (int idx = tid; idx < n * DK; idx += kThreads) {
            const int t = idx / DK, c = idx % DK;
            const size_t o = (((size_t)b * a.L + t0 + t) * a.H + h) * DK + c;
            a.dq[o] = Gq[idx];
            a.dk[o] = Gk[idx];
        }
        for (int idx = tid; idx < n * DV; idx += kThreads) {
            const int t = idx / DV, c = idx % DV;
            a.dv[(((size_t)b * a.L + t0 + t) * a.H + h) * DV + c] = sc.be[t] * dR[idx];
        }
        if (tid < n) {
            const size_t row = ((size_t)b * a.L + t0 + tid) * a.H + h;
            a.dbeta[row] = red[tid][0];
            a.dalpha[row] = red[tid][3] / sc.al[tid];
        }
        __syncthreads();
    }
}

template <typename T, int DK, int DV>
cudaError_t run_all(const GdnBwdArgs &a, cudaStream_t s) {
    constexpr size_t fs = fscan_smem_floats<DK, DV>() * sizeof(float);
    constexpr size_t ds = dscan_smem_floats<DK, DV>() * sizeof(float);
    static_assert(fs <= 232448 && ds <= 232448, "scan shared memory exceeds 227 KB");
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(gdn_bwd_fscan<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fs);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn_bwd_dscan<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ds);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    gdn_bwd_prep<T, DK, DV><<<a.grid_chunks, kThreads, 0, s>>>(a);
    gdn_bwd_fscan<DK, DV><<<dim3(DV / kScanRows, a.B * a.H), kThreads, fs, s>>>(a);
    gdn_bwd_dscan<DK, DV><<<dim3(DV / kScanRows, a.B * a.H), kThreads, ds, s>>>(a);
    gdn_bwd_local<T, DK, DV><<<a.grid_chunks, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t gdn_bwd_ws_floats(int d_k, int d_v) {
    // the larger of the prep and local kernels' per-CTA workspaces
    const size_t prep = (size_t)kC * (4 * d_k + 3 * d_v) + 2 * kC * kC;
    const size_t local = (size_t)kC * (2 * d_k + 2 * d_v) + 5 * kC * kC + 5 * (size_t)kC * d_v +
                         2 * (size_t)kC * d_k + (size_t)kC * (d_k > d_v ? d_k : d_v);
    return prep > local ? prep : local;
}

cudaError_t launch_gdn_bwd(const GdnBwdArgs &a, bool bf16, cudaStream_t s) {
    if ((long long)a.B * a.L * a.H == 0) return cudaSuccess;
#define HLTA_GDN_BWD(DK, DV)                                                                  \
    if (a.d_k == DK && a.d_v == DV)                                                           \
        return bf16 ? run_all<__nv_bfloat16, DK, DV>(a, s) : run_all<float, DK, DV>(a, s);
    HLTA_GDN_BWD(128, 128)
    HLTA_GDN_BWD(64, 64)
    HLTA_GDN_BWD(128, 64)
    HLTA_GDN_BWD(64, 128)
#undef HLTA_GDN_BWD
    return cudaErrorInvalidValue;
}

}  // namespace hlta
