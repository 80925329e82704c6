// tc_gdn.cu -- chunked gated delta memory on the sm_100a tensor cores (bf16 in).
//
// Kairos paper, section 2.2.1: S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T)
// + beta_t v_t k_t^T and o_t = S_t q_t (retrieval from the decayed state).
// The recurrence is regrouped into chunks of C = 64 tokens (a derivation, not on
// the pages).  Inside a chunk with start state S0, l_t = sum_{s<=t} log alpha_s,
// g_t = exp(l_t) and u_t = beta_t (v_t - alpha_t S_{t-1} k_t):
//   (I + A) U = diag(beta) V - diag(beta g) K S0^T,  A_ts = beta_t e^{l_t-l_s} k_t.k_s (s < t)
//   T = (I + A)^-1,  W = T diag(beta g) K,  U~ = T diag(beta) V,  U = U~ - W S0^T
//   O = diag(g) Q S0^T + Pm U,                Pm_ts = e^{l_t-l_s} q_t.k_s (s <= t)
//   S_C = g_C S0 + U^T diag(e^{l_C-l}) K.
// The update form printed as Eq. (2)/(6), u_t = beta_t (v_t - S_{t-1} k_t), is the
// same system with l_t replaced by l_{t-1} in A's rows and in W's factors
// (HLTA_GDN_PAGES).
// Two kernels:
//   gdn_prep_kernel  (one CTA per chunk, all chunks in parallel): [K;Q] K^T on
//       tcgen05 (bf16), the decay masks, T by blocked forward substitution on
//       CUDA cores (16x16 diagonal blocks, then the block diagonals below), then
//       W^T = K^T (T diag(beta g))^T and U~^T = V^T (T diag(beta))^T as fp16
//       tcgen05 MMAs.  Writes W and g*Q (fp16), K (fp16), Pm (fp16), U~ (fp32)
//       and l to a per-chunk scratch.
//   gdn_scan_kernel  (one CTA per (b, h), chunks in sequence): the d_v = 128 rows
//       of the state are the MMA's M dimension.  Per chunk the serial chain is
//         S0 W^T = S16 W^T                 (S16: fp16 copy of S in TMEM)
//         U^T = U~^T - S0 W^T               (CUDA cores, fp32)
//         D = U^T (diag(e^{l_C-l}) K)        (A operand read from TMEM)
//         S = g_C S + D  (fp32, held in the math warps' registers), S16 = fp16(S)
//       and the output half runs beside it: O^T = S16 (gQ)^T + U^T Pm^T, written
//       per token.
// Internal operands are fp16 (11-bit mantissa) with fp32 accumulation; every
// value they carry is bounded (unit keys, alpha in (0,1], beta in [0,1]).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <string.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tc_gdn.h"

namespace hlta {

namespace {

using namespace sm100;

constexpr int kC = 64;     // chunk
constexpr int kD = 128;    // d_k = d_v
// scratch per chunk
constexpr size_t kWQBytes = 128 * kD * 2;   // [W; gQ] fp16, 128 rows
constexpr size_t kK16Bytes = kC * kD * 2;   // K fp16
constexpr size_t kPmBytes = kC * kC * 2;    // Pm fp16
constexpr size_t kUtBytes = kC * kD * 4;    // U~ fp32
constexpr size_t kEllBytes = 2 * kC * 4;  // l_t and e^{l_C - l_t}

struct GdnScratch {
    __half *wq;   // [BH * NC * 128][128]
    __half *k16;  // [BH * NC * 64][128]: e^{l_C - l_t} k_t
    __half *pm;   // [BH * NC * 64][64]
    float *ut;    // [BH * NC * 64][128]
    float *ell;   // [BH * NC][128]: l_t, then e^{l_C - l_t}
};

// =====================================================================
// prep
// =====================================================================
struct PrepParams {
    const float *alpha, *beta;  // [B, L, H]
    int L, H, NC;
    int c_begin;                // first chunk of this launch (blockIdx.x is relative)
    int form;                   // HLTA_GDN_DECAYED / HLTA_GDN_PAGES
    GdnScratch scr;
    int *dev_err;
};

struct __align__(1024) PrepSmem {
    // 2 regions (d 0-63 / 64-127) x 128 rows: rows 0-63 K, 64-127 Q.  Once Q has
    // been read, its rows hold the B operands (T diag(beta g))[t][s] (region 0)
    // and (T diag(beta))[t][s] (region 1), fp16, K-major.
    uint8_t kq[32768];
    uint8_t v[16384];    // 2 regions x 64 rows of V
    float A[kC][kC + 4];  // rows padded to 16 bytes; T^T is built in the upper triangle
    float ell[kC], beta[kC], gam[kC], dec[kC];
    float ellr[kC], gamr[kC];  // log-decay / decay that token t's retrieval sees (see below)
    uint64_t bar_tma, bar_mma1, bar_mma2;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t sw128_off(int row, int chunk16) {
    // byte offset of 16-byte chunk `chunk16` (0..7) of row `row` in a 128B-swizzled tile
    return (uint32_t)(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(128, 3)
gdn_prep_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const PrepParams p) {
    extern __shared__ uint8_t smem_raw[];
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = p.c_begin + blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const size_t chunk_id = (size_t)bh * p.NC + c;
    const int t0 = c * kC;
    volatile int *abort = &sm.abort;

    // alpha and beta of the chunk's tokens (tokens past the end act as alpha = 1,
    // beta = 0): the loads are in flight during the setup below
    float al = 1.f, be = 0.f;
    if (tid < kC && t0 + tid < p.L) {
        const size_t i = ((size_t)b * p.L + t0 + tid) * p.H + h;
        al = p.alpha[i];
        be = p.beta[i];
    }
    if (tid == 0) {
        sm.abort = *reinterpret_cast<volatile int *>(p.dev_err) != 0 ? 1 : 0;
        mbar_init(&sm.bar_tma, 1);
        mbar_init(&sm.bar_mma1, 1);
        mbar_init(&sm.bar_mma2, 1);
        fence_barrier_init();
    }
    // 128 columns: [K; Q] K^T in 0-63, later W^T in 0-63 and U~^T in 64-127, so
    // that four CTAs of this kernel fit one SM's tensor memory
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);

    if (tid == 0 && !*abort) {
        mbar_expect_tx(&sm.bar_tma, 32768 + 16384);
        tma_load_4d(sm.kq, &tmK, 0, h, t0, b, &sm.bar_tma);
        tma_load_4d(sm.kq + 8192, &tmQ, 0, h, t0, b, &sm.bar_tma);
        tma_load_4d(sm.kq + 16384, &tmK, 64, h, t0, b, &sm.bar_tma);
        tma_load_4d(sm.kq + 24576, &tmQ, 64, h, t0, b, &sm.bar_tma);
        tma_load_4d(sm.v, &tmV, 0, h, t0, b, &sm.bar_tma);
        tma_load_4d(sm.v + 8192, &tmV, 64, h, t0, b, &sm.bar_tma);
    }
    // decay prefix
    if (tid < kC) {
        float x = logf(al);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        sm.ell[tid] = x;  // warp-local prefix; warp 1 adds warp 0's total below
        sm.beta[tid] = be;
    }
    __syncthreads();
    if (tid >= 32 && tid < kC) sm.ell[tid] += sm.ell[31];
    __syncthreads();
    if (tid < kC) {
        sm.gam[tid] = expf(sm.ell[tid]);
        sm.dec[tid] = expf(sm.ell[kC - 1] - sm.ell[tid]);
        // The retrieval of token t reads alpha_t S_{t-1} (decayed form: l_t) or
        // S_{t-1} (the printed Eq. (2)/(6): l_{t-1}, 0 for the chunk's first
        // token).  Only A's rows and W's factors depend on it; with
        // beta'_t = beta_t / alpha_t the printed form is the decayed form, and
        // forming e^{l_{t-1} - l_s} directly keeps every factor <= 1.
        sm.ellr[tid] = p.form == HLTA_GDN_PAGES ? (tid == 0 ? 0.f : sm.ell[tid - 1]) : sm.ell[tid];
        sm.gamr[tid] = expf(sm.ellr[tid]);
        p.scr.ell[chunk_id * 2 * kC + tid] = sm.ell[tid];
        p.scr.ell[chunk_id * 2 * kC + kC + tid] = sm.dec[tid];
    }

    // [K; Q] K^T -> TMEM cols 0..63 (bf16 operands, exact products)
    if (tid == 0) {
        if (!*abort && mbar_wait(&sm.bar_tma, 0, abort, p.dev_err)) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
            const uint32_t base = smem_u32(sm.kq);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                umma_ss(tmem, smem_desc_sw128(base + off, 16, 1024), smem_desc_sw128(base + off, 16, 1024),
                        idesc, kk > 0 ? 1u : 0u);
            }
            umma_commit(&sm.bar_mma1);
        }
    }
    __syncthreads();  // ell / beta / gam visible
    const bool ok1 = __all_sync(0xffffffffu, !*abort && mbar_wait(&sm.bar_mma1, 0, abort, p.dev_err));
    if (ok1) {
        tc_fence_after();
        uint32_t g0[32], g1[32];
        tmem_ld32(tl, g0);
        tmem_ld32(tl + 32, g1);
        tmem_wait_ld();
        if (tid < kC) {
            const int t = tid;
            const float lt = sm.ellr[t], bt = sm.beta[t];
#pragma unroll
            for (int s = 0; s < kC; s += 4) {
                float a[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float gs = __uint_as_float(s + e < 32 ? g0[s + e] : g1[s + e - 32]);
                    a[e] = (s + e < t) ? bt * __expf(lt - sm.ell[s + e]) * gs : 0.f;
                }
                *reinterpret_cast<float4 *>(&sm.A[t][s]) = make_float4(a[0], a[1], a[2], a[3]);
            }
        } else {
            const int t = tid - kC;
            const float lt = sm.ell[t];
            uint32_t w[32];
#pragma unroll
            for (int s = 0; s < kC; s += 2) {
                const float q0 = __uint_as_float(s < 32 ? g0[s] : g1[s - 32]);
                const float q1 = __uint_as_float(s + 1 < 32 ? g0[s + 1] : g1[s + 1 - 32]);
                const float p0 = (s <= t) ? __expf(lt - sm.ell[s]) * q0 : 0.f;
                const float p1 = (s + 1 <= t) ? __expf(lt - sm.ell[s + 1]) * q1 : 0.f;
                w[s / 2] = pack_f16x2(p0, p1);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(p.scr.pm + (chunk_id * kC + t) * kC);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
    }
    tc_fence_before();  // the TMEM reads above precede the MMA that reuses columns 0-63
    __syncthreads();

    if (!*abort) {
        // bf16 -> fp16 in place (the fp16 MMA below takes K and V), the scan's
        // copies of K (carrying the decay to the chunk end) and of g*Q
        for (int i = tid; i < 2 * 128 * 8; i += 128) {
            const int region = i >> 10, row = (i >> 3) & 127, ch = i & 7;
            const uint32_t off = region * 16384 + sw128_off(row, ch);
            uint4 *ptr = reinterpret_cast<uint4 *>(sm.kq + off);
            const uint4 raw = *ptr;
            const int dcol = region * 64 + ch * 8;
            if (row < kC) {
                *ptr = bf16x8_to_f16x8(raw, 1.f);
                *reinterpret_cast<uint4 *>(p.scr.k16 + (chunk_id * kC + row) * kD + dcol) =
                    bf16x8_to_f16x8(raw, sm.dec[row]);
            } else {
                *reinterpret_cast<uint4 *>(p.scr.wq + (chunk_id * 128 + row) * kD + dcol) =
                    bf16x8_to_f16x8(raw, sm.gam[row - kC]);
            }
        }
        for (int i = tid; i < 2 * kC * 8; i += 128) {
            const int region = i >> 9, row = (i >> 3) & 63, ch = i & 7;
            uint4 *ptr = reinterpret_cast<uint4 *>(sm.v + region * 8192 + sw128_off(row, ch));
            *ptr = bf16x8_to_f16x8(*ptr, 1.f);
        }
        // T = (I + A)^-1, blocked by 16: the diagonal blocks by forward
        // substitution, then the block diagonals below them in turn,
        //   T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj   (i > j).
        // A is strictly lower triangular; T is kept transposed in the upper
        // triangle (diagonal included) of the same array: T[t][s] at A[s][t].
        if (tid < kC) {
            const int bi = tid >> 4, c = tid & 15, o = bi * 16;
            float x[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                float acc = (t == c) ? 1.f : 0.f;
#pragma unroll
                for (int q = 0; q < t; ++q) acc = fmaf(-sm.A[o + t][o + q], x[q], acc);
                x[t] = (t < c) ? 0.f : acc;
            }
#pragma unroll
            for (int t = 0; t < 16; ++t)
                if (t >= c) sm.A[o + c][o + t] = x[t];
        }
        __syncthreads();
        // Block diagonal d: one thread per column c of each block (i, j = i - d).
        // It forms y = sum_k A_ik T_kj[:, c] (16 values), then
        // T_ij[:, c] = -T_ii y, with sixteen independent accumulators each time.
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {
            if (tid < (4 - d) * 16) {
                const int j = tid >> 4, i = j + d, c = tid & 15;
                float y[16];
#pragma unroll
                for (int mrow = 0; mrow < 16; ++mrow) y[mrow] = 0.f;
                for (int k = j; k < i; ++k) {
                    // T_kj[n][c] sits at A[16j + c][16k + n]; in the diagonal block
                    // (k == j) the entries n < c of that row are A's, not T's (zero)
                    float tc[16];
#pragma unroll
                    for (int n = 0; n < 16; n += 4) {
                        const float4 t4 = *reinterpret_cast<const float4 *>(&sm.A[16 * j + c][16 * k + n]);
                        tc[n] = t4.x;
                        tc[n + 1] = t4.y;
                        tc[n + 2] = t4.z;
                        tc[n + 3] = t4.w;
                    }
                    if (k == j) {
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            if (n < c) tc[n] = 0.f;
                    }
#pragma unroll
                    for (int mrow = 0; mrow < 16; ++mrow) {
#pragma unroll
                        for (int n = 0; n < 16; n += 4) {
                            const float4 a4 = *reinterpret_cast<const float4 *>(&sm.A[16 * i + mrow][16 * k + n]);
                            y[mrow] = fmaf(a4.x, tc[n], y[mrow]);
                            y[mrow] = fmaf(a4.y, tc[n + 1], y[mrow]);
                            y[mrow] = fmaf(a4.z, tc[n + 2], y[mrow]);
                            y[mrow] = fmaf(a4.w, tc[n + 3], y[mrow]);
                        }
                    }
                }
                // T_ij[r][c] = -sum_{m <= r} T_ii[r][m] y[m]; T_ii[r][m] sits at A[16i + m][16i + r]
                float tr[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) tr[r] = 0.f;
#pragma unroll
                for (int mrow = 0; mrow < 16; ++mrow) {
#pragma unroll
                    for (int r = 0; r < 16; r += 4) {
                        if (r + 3 < mrow) continue;
                        const float4 t4 = *reinterpret_cast<const float4 *>(&sm.A[16 * i + mrow][16 * i + r]);
                        if (r >= mrow) tr[r] = fmaf(t4.x, y[mrow], tr[r]);
                        if (r + 1 >= mrow) tr[r + 1] = fmaf(t4.y, y[mrow], tr[r + 1]);
                        if (r + 2 >= mrow) tr[r + 2] = fmaf(t4.z, y[mrow], tr[r + 2]);
                        if (r + 3 >= mrow) tr[r + 3] = fmaf(t4.w, y[mrow], tr[r + 3]);
                    }
                }
#pragma unroll
                for (int r = 0; r < 16; r += 4)
                    *reinterpret_cast<float4 *>(&sm.A[16 * j + c][16 * i + r]) =
                        make_float4(-tr[r], -tr[r + 1], -tr[r + 2], -tr[r + 3]);
            }
            __syncthreads();
        }
        // B operands of the fp16 MMA, K-major rows t over the Q rows of kq:
        // (T diag(beta g))[t][s] in region 0, (T diag(beta))[t][s] in region 1
        {
            const int t = tid & 63;
            const bool second = tid >= 64;
            __half *dst = reinterpret_cast<__half *>(sm.kq + (second ? 16384 : 0) + 8192);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const int s0 = ch * 8 + e, s1 = s0 + 1;
                    const float f0 = second ? sm.beta[s0] : sm.beta[s0] * sm.gamr[s0];
                    const float f1 = second ? sm.beta[s1] : sm.beta[s1] * sm.gamr[s1];
                    const float t0 = s0 <= t ? sm.A[s0][t] : 0.f;
                    const float t1 = s1 <= t ? sm.A[s1][t] : 0.f;
                    w[e / 2] = pack_f16x2(t0 * f0, t1 * f1);
                }
                *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(dst) + sw128_off(t, ch)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        fence_proxy_async_smem();
    }
    __syncthreads();

    // W^T = K^T (T diag(beta g))^T -> cols 0..63; U~^T = V^T (T diag(beta))^T -> cols 64..127
    if (tid == 0 && !*abort) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 64, 1, 0);
        const uint32_t kb = smem_u32(sm.kq), vb = smem_u32(sm.v);
        const uint32_t b1 = smem_u32(sm.kq + 8192), b2 = smem_u32(sm.kq + 16384 + 8192);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            umma_ss(tmem, smem_desc_sw128(kb + kk * 2048, 16384, 1024), smem_desc_sw128(b1 + kk * 32, 16, 1024),
                    idesc, kk > 0 ? 1u : 0u);
            umma_ss(tmem + 64, smem_desc_sw128(vb + kk * 2048, 8192, 1024), smem_desc_sw128(b2 + kk * 32, 16, 1024),
                    idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.bar_mma2);
    }
    const bool ok2 = __all_sync(0xffffffffu, !*abort && mbar_wait(&sm.bar_mma2, 0, abort, p.dev_err));
    if (ok2) {
        tc_fence_after();
        const int r = tid;  // d_k index for W^T, d_v index for U~^T
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t w[32], u[32];
            tmem_ld32(tl + half * 32, w);
            tmem_ld32(tl + 64 + half * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int t = half * 32 + j;
                p.scr.wq[(chunk_id * 128 + t) * kD + r] = __float2half_rn(__uint_as_float(w[j]));
                p.scr.ut[(chunk_id * kC + t) * kD + r] = __uint_as_float(u[j]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// =====================================================================
// scan
// =====================================================================
struct ScanParams {
    int L, H, NC;
    int c_begin, nseg;  // this launch scans chunks [c_begin, c_begin + nseg)
    const float *S_in;
    float *S_out;
    const float *gates;
    int out_mode;
    int out_tma;  // 0: per-token stores; 1: TMA store of fp32 tiles (acc); 2: TMA reduce-add (acc);
                  // 3: TMA store of bf16 tiles (out)
    float *acc;
    __nv_bfloat16 *out;
    int *dev_err;
};

constexpr uint32_t kStageTx = (uint32_t)(kWQBytes + kK16Bytes + kPmBytes + kUtBytes + kEllBytes);

struct __align__(1024) ScanStage {
    uint8_t wq[kWQBytes];    // 2 regions x 128 rows, K-major SW128
    uint8_t k16[kK16Bytes];  // 2 regions x 64 rows (d 0-63 / 64-127)
    uint8_t pm[kPmBytes];    // 64 rows x 64, SW128
    float ut[kC * kD];       // [t][dv] fp32, unswizzled
    float ell[2 * kC];       // l_t, then e^{l_C - l_t}
};

struct __align__(1024) ScanSmem {
    ScanStage st[2];
    uint8_t ostage[kC * kD * 4];  // one chunk of outputs [token][d_v], fp32 or bf16, for the TMA store
    uint64_t full[2], empty[2], bar_p1, bar_u, bar_d, bar_o, bar_s16, bar_oread, bar_sfree, bar_sfull;
    uint32_t tmem_base;
    int abort;
};

static_assert(sizeof(ScanSmem) + 1024 <= 232448, "scan shared memory exceeds the 227 KB per-block limit");

// TMEM columns of the scan
constexpr uint32_t kP1 = 0;     // [S0 W^T | S0 (gQ)^T]  -> O accumulates on cols 64..127
constexpr uint32_t kU = 128;    // U^T fp16 (32 cols)
constexpr uint32_t kS16 = 192;  // fp16 copy of S (64 cols)
constexpr uint32_t kDS = 256;   // U^T (diag(e^{l_C - l}) K)

constexpr int kScanThreads = 320;  // producer, MMA issuer, 8 math warps

__global__ void __launch_bounds__(kScanThreads, 1)
gdn_scan_kernel(const __grid_constant__ CUtensorMap tmWQ, const __grid_constant__ CUtensorMap tmK16,
                const __grid_constant__ CUtensorMap tmPm, const __grid_constant__ CUtensorMap tmUt,
                const __grid_constant__ CUtensorMap tmEll, const __grid_constant__ CUtensorMap tmOut,
                const ScanParams p) {
    extern __shared__ uint8_t smem_raw[];
    ScanSmem &sm = *reinterpret_cast<ScanSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, b = blockIdx.y;
    const int bh = b * p.H + h;
    const int NC = p.nseg;  // chunks of this launch; chunk c here is p.c_begin + c
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        sm.abort = *reinterpret_cast<volatile int *>(p.dev_err) != 0 ? 1 : 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1 + 256);
        }
        mbar_init(&sm.bar_p1, 1);
        mbar_init(&sm.bar_u, 256);
        mbar_init(&sm.bar_d, 1);
        mbar_init(&sm.bar_o, 1);
        mbar_init(&sm.bar_s16, 256);
        mbar_init(&sm.bar_oread, 256);
        mbar_init(&sm.bar_sfree, 1);
        mbar_init(&sm.bar_sfull, 256);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&tmWQ);
            prefetch_tensormap(&tmK16);
            prefetch_tensormap(&tmPm);
            prefetch_tensormap(&tmUt);
            prefetch_tensormap(&tmEll);
            int issued = 0;
            for (int c = 0; c < NC && !*abort; ++c) {
                const int s = c & 1;
                if (c >= 2 && !mbar_wait(&sm.empty[s], ((c >> 1) - 1) & 1, abort, p.dev_err)) break;
                ScanStage &st = sm.st[s];
                const int cid = bh * p.NC + p.c_begin + c;
                mbar_expect_tx(&sm.full[s], kStageTx);
                tma_load_2d(st.wq, &tmWQ, 0, cid * 128, &sm.full[s]);
                tma_load_2d(st.wq + 16384, &tmWQ, 64, cid * 128, &sm.full[s]);
                tma_load_2d(st.k16, &tmK16, 0, cid * kC, &sm.full[s]);
                tma_load_2d(st.k16 + 8192, &tmK16, 64, cid * kC, &sm.full[s]);
                tma_load_2d(st.pm, &tmPm, 0, cid * kC, &sm.full[s]);
                tma_load_2d(st.ut, &tmUt, 0, cid * kC, &sm.full[s]);
                tma_load_2d(st.ell, &tmEll, 0, cid, &sm.full[s]);
                issued = c + 1;
            }
            if (*abort) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                for (int c = (issued > 2 ? issued - 2 : 0); c < issued; ++c)
                    mbar_wait(&sm.full[c & 1], (c >> 1) & 1, no_abort, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // Per chunk, the serial chain is S0 W^T -> U -> U^T K -> S.  The output
            // half (S0 (gQ)^T + U Pm^T, into columns 64-127 of P1) is issued
            // beside it; it may only overwrite P1's columns 64-127 once the
            // previous chunk's output has been read from them.
            const uint32_t idh = idesc_f16_f32(128, 64, 0, 0);
            const uint32_t id3 = idesc_f16_f32(128, 128, 0, 1);
            int committed = 0;
            for (int c = 0; c < NC; ++c) {
                const int s = c & 1;
                ScanStage &st = sm.st[s];
                if (!mbar_wait(&sm.full[s], (c >> 1) & 1, abort, p.dev_err)) break;
                if (!mbar_wait(&sm.bar_s16, c & 1, abort, p.dev_err)) break;
                tc_fence_after();
                const uint32_t wq = smem_u32(st.wq);
                // S0 W^T (rows 0-63 of [W; gQ])
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tmem + kP1, tmem + kS16 + kk * 8,
                            smem_desc_sw128(wq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), idh,
                            kk > 0 ? 1u : 0u);
                umma_commit(&sm.bar_p1);
                // S0 (gQ)^T (rows 64-127), reading S16 before the state update rewrites it
                if (c > 0 && !mbar_wait(&sm.bar_oread, (c - 1) & 1, abort, p.dev_err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tmem + kP1 + 64, tmem + kS16 + kk * 8,
                            smem_desc_sw128(wq + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32, 16, 1024), idh,
                            kk > 0 ? 1u : 0u);
                if (!mbar_wait(&sm.bar_u, c & 1, abort, p.dev_err)) break;
                tc_fence_after();
                const uint32_t pm = smem_u32(st.pm), k16 = smem_u32(st.k16);
                // D = U^T (diag(e^{l_C - l}) K): the state update waits only for this
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_ts(tmem + kDS, tmem + kU + kk * 8, smem_desc_sw128(k16 + kk * 2048, 8192, 1024), id3,
                            kk > 0 ? 1u : 0u);
                umma_commit(&sm.bar_d);
                // O^T += U^T Pm^T
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_ts(tmem + kP1 + 64, tmem + kU + kk * 8, smem_desc_sw128(pm + kk * 32, 16, 1024), idh, 1u);
                umma_commit(&sm.bar_o);
                umma_commit(&sm.empty[s]);
                committed = c + 1;
            }
            if (*abort && committed) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                mbar_wait(&sm.bar_o, (committed - 1) & 1, no_abort, nullptr);
            }
        }
    } else {
        // math warps: two groups of four; thread = row of S (d_v index) = TMEM lane.
        // Group w takes tokens [32w, 32w+32) of U and O and d_k columns
        // [64w, 64w+64) of the state, which it keeps in fp32 registers.
        const int w = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const float gate = p.gates[h * 3 + 2];
        float S[64];
        {
            const float *src = p.S_in ? p.S_in + ((size_t)bh * kD + row) * kD + 64 * w : nullptr;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 x = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0, 0, 0, 0);
                S[j] = x.x;
                S[j + 1] = x.y;
                S[j + 2] = x.z;
                S[j + 3] = x.w;
            }
            uint32_t f16w[32];
#pragma unroll
            for (int j = 0; j < 64; j += 2) f16w[j / 2] = pack_f16x2(S[j], S[j + 1]);
            tmem_st32(tl + kS16 + 32 * w, f16w);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_s16);
        }
        bool ok = true;
        for (int c = 0; c < NC && ok; ++c) {
            const int s = c & 1;
            ScanStage &st = sm.st[s];
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[s], (c >> 1) & 1, abort, p.dev_err) &&
                                             mbar_wait(&sm.bar_p1, c & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float gC = __expf(st.ell[kC - 1]);
            // U = U~ - S0 W^T for tokens [32w, 32w+32) of this row of U^T
            {
                uint32_t x[32], u[16];
                tmem_ld32(tl + kP1 + 32 * w, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const int t = 32 * w + j;
                    u[j / 2] = pack_f16x2(st.ut[t * kD + row] - __uint_as_float(x[j]),
                                          st.ut[(t + 1) * kD + row] - __uint_as_float(x[j + 1]));
                }
                tmem_st16(tl + kU + 16 * w, u);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&sm.bar_u);
            mbar_arrive(&sm.empty[s]);  // done with this stage's U~ and l
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_d, c & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // S = g_C S + U^T (diag(e^{l_C - l}) K) on columns [64w, 64w+64); S16 = fp16(S)
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                uint32_t d[32], f16w[16];
                tmem_ld32(tl + kDS + 64 * w + 32 * q2, d);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    float &s0 = S[32 * q2 + j], &s1 = S[32 * q2 + j + 1];
                    s0 = fmaf(gC, s0, __uint_as_float(d[j]));
                    s1 = fmaf(gC, s1, __uint_as_float(d[j + 1]));
                    f16w[j / 2] = pack_f16x2(s0, s1);
                }
                tmem_st16(tl + kS16 + 32 * w + 16 * q2, f16w);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_s16);
            // O for tokens [32w, 32w+32): read it, then free its columns for the
            // next chunk's S0 (gQ)^T
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_o, c & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t o[32];
            tmem_ld32(tl + kP1 + 64 + 32 * w, o);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_oread);
            if (p.out_tma) {
                // the chunk's outputs go through shared memory and one TMA store,
                // issued by warp 2 once all eight warps have written their tokens
                const bool elect = warp == 2 && lane == 0;
                if (elect) {
                    if (c > 0) bulk_wait_read0();  // the previous chunk's tile has been read
                    mbar_arrive(&sm.bar_sfree);
                }
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfree, c & 1, abort, p.dev_err))) {
                    ok = false;
                    break;
                }
                if (p.out_tma == 3) {
                    __nv_bfloat16 *st16 = reinterpret_cast<__nv_bfloat16 *>(sm.ostage);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        st16[(32 * w + t) * kD + row] = __float2bfloat16_rn(gate * __uint_as_float(o[t]));
                } else {
                    float *st32 = reinterpret_cast<float *>(sm.ostage);
#pragma unroll
                    for (int t = 0; t < 32; ++t) st32[(32 * w + t) * kD + row] = gate * __uint_as_float(o[t]);
                }
                fence_proxy_async_smem();
                mbar_arrive(&sm.bar_sfull);
                if (warp == 2) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull, c & 1, abort, p.dev_err))) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        const int tok0 = (p.c_begin + c) * kC;  // rows past L are clipped by the TMA unit
                        if (p.out_tma == 2)
                            tma_reduce_add_4d(&tmOut, sm.ostage, 0, h, tok0, b);
                        else
                            tma_store_4d(&tmOut, sm.ostage, 0, h, tok0, b);
                        bulk_commit();
                    }
                }
                continue;
            }
            // outputs of tokens [32w, 32w+32) of this chunk, column `row`, in groups
            // of 8 tokens whose accumulator loads are issued before their stores
            const int t0 = (p.c_begin + c) * kC + 32 * w;
            const int nt = min(32, p.L - t0);
            const size_t stride = (size_t)p.H * kD;
            const size_t idx0 = (((size_t)b * p.L + t0) * p.H + h) * kD + row;
            const bool add = p.out_mode == OUT_ADD || p.out_mode == OUT_FINAL;
            const bool to_acc = p.out_mode == OUT_STORE || p.out_mode == OUT_ADD;
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = 8 * g8 + e;
                    v8[e] = gate * __uint_as_float(o[t]);
                    if (add && t < nt) v8[e] += p.acc[idx0 + t * stride];
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = 8 * g8 + e;
                    if (t >= nt) continue;
                    if (to_acc)
                        p.acc[idx0 + t * stride] = v8[e];
                    else
                        p.out[idx0 + t * stride] = __float2bfloat16_rn(v8[e]);
                }
            }
        }
        if (warp == 2 && lane == 0) bulk_wait0();  // stores in flight complete before exit
        if (ok && p.S_out) {
            float *dst = p.S_out + ((size_t)bh * kD + row) * kD + 64 * w;
#pragma unroll
            for (int j = 0; j < 64; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// =====================================================================
// host side
// =====================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

bool map_2d(CUtensorMap *m, CUtensorMapDataType dt, size_t esize, const void *base, uint64_t cols, uint64_t rows,
            uint32_t box_c, uint32_t box_r, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * esize};
    const cuuint32_t box[2] = {box_c, box_r};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D view (d, H, L, B) of a [B, L, H, 128] bf16 tensor, box (64, 1, 64, 1).
bool map_tokens(CUtensorMap *m, const void *base, int H, int L, int B) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)L * H * kD * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output tiles of the scan: 4-D view (d_v, H, L, B) of a [B, L, H, 128] fp32 or
// bf16 tensor, box (128, 1, 64, 1) -- one chunk of one head.
bool map_out(CUtensorMap *m, const void *base, bool bf16, int H, int L, int B) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || !base) return false;
    const size_t es = bf16 ? 2 : 4;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * es, (cuuint64_t)H * kD * es, (cuuint64_t)L * H * kD * es};
    const cuuint32_t box[4] = {kD, 1, kC, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void *>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// How the scan writes its outputs for an output mode (ScanParams::out_tma), with
// the tensor map it needs; per-token stores when no TMA form applies.
int scan_out_tma(CUtensorMap *m, int mode, float *acc, void *out, int H, int L, int B) {
    memset(m, 0, sizeof(*m));
    if ((mode == OUT_STORE || mode == OUT_ADD) && map_out(m, acc, false, H, L, B)) return mode == OUT_STORE ? 1 : 2;
    if (mode == OUT_FINAL_ONLY && map_out(m, out, true, H, L, B)) return 3;
    memset(m, 0, sizeof(*m));
    return 0;
}

class TcGdnImpl : public TcGdn {
public:
    TcGdnImpl(const hlta_config &c, int max_nc) : cfg_(c), max_nc_(max_nc) {}
    ~TcGdnImpl() override {
        cudaFree(base_);
        cudaFree(s_mid_);
        if (prep_stream_) cudaStreamDestroy(prep_stream_);
        for (auto e : ev_) if (e) cudaEventDestroy(e);
    }

    bool init() {
        const size_t n = (size_t)cfg_.B * cfg_.H * max_nc_;
        bytes_ = n * (kWQBytes + kK16Bytes + kPmBytes + kUtBytes + kEllBytes);
        const size_t sbytes = (size_t)cfg_.B * cfg_.H * kD * kD * sizeof(float);
        int prio_lo = 0, prio_hi = 0;
        cudaDeviceGetStreamPriorityRange(&prio_lo, &prio_hi);
        bool ok = cudaMalloc(&base_, bytes_) == cudaSuccess && cudaMalloc(&s_mid_, 2 * sbytes) == cudaSuccess &&
                  cudaStreamCreateWithPriority(&prep_stream_, cudaStreamNonBlocking, prio_hi) == cudaSuccess;
        for (auto &e : ev_) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) cudaGetLastError();
        return ok;
    }

    bool covers(int L) const override { return L >= kC && (L + kC - 1) / kC <= max_nc_; }

    cudaError_t run(const void *q, const void *k, const void *v, const float *alpha, const float *beta, int L,
                    const float *S_in, float *S_out, const float *gates, int mode, float *acc, void *out,
                    int *dev_err, cudaStream_t s, bool *done, int *launches) override {
        *done = false;
        if (L < kC) return cudaSuccess;  // shorter than one chunk: recurrent kernel
        const int NC = (L + kC - 1) / kC;
        if (NC > max_nc_) return cudaSuccess;
        const int BH = cfg_.B * cfg_.H;
        GdnScratch scr;
        char *p = static_cast<char *>(base_);
        const size_t n = (size_t)BH * NC;
        scr.wq = reinterpret_cast<__half *>(p);
        p += n * kWQBytes;
        scr.k16 = reinterpret_cast<__half *>(p);
        p += n * kK16Bytes;
        scr.pm = reinterpret_cast<__half *>(p);
        p += n * kPmBytes;
        scr.ut = reinterpret_cast<float *>(p);
        p += n * kUtBytes;
        scr.ell = reinterpret_cast<float *>(p);

        CUtensorMap mq, mk, mv, mwq, mk16, mpm, mut, mell;
        if (!map_tokens(&mq, q, cfg_.H, L, cfg_.B) || !map_tokens(&mk, k, cfg_.H, L, cfg_.B) ||
            !map_tokens(&mv, v, cfg_.H, L, cfg_.B) ||
            !map_2d(&mwq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, scr.wq, kD, n * 128, 64, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
            !map_2d(&mk16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, scr.k16, kD, n * kC, 64, kC,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
            !map_2d(&mpm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, scr.pm, kC, n * kC, 64, kC,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
            !map_2d(&mut, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, scr.ut, kD, n * kC, kD, kC,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !map_2d(&mell, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, scr.ell, 2 * kC, n, 2 * kC, 1,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;

        const size_t prep_smem = sizeof(PrepSmem) + 1024, scan_smem = sizeof(ScanSmem) + 1024;
        if (!attr_set_) {
            cudaError_t e = cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)prep_smem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)scan_smem);
            if (e != cudaSuccess) return e;
            attr_set_ = true;
        }
        // The chunks are cut into up to kSegs segments.  The prep of segment g+1
        // runs on an internal stream while the scan of segment g runs on `s`;
        // the scans carry the state through a small handle-owned buffer.
        const int segs = NC >= 4 * kSegs ? kSegs : (NC >= 8 ? 2 : 1);
        const int per = (NC + segs - 1) / segs;
        const size_t sstride = (size_t)BH * kD * kD;
        cudaError_t e = cudaEventRecord(ev_[0], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(prep_stream_, ev_[0], 0);
        PrepParams pp;
        pp.alpha = alpha;
        pp.beta = beta;
        pp.L = L;
        pp.H = cfg_.H;
        pp.NC = NC;
        pp.form = cfg_.gdn_form;
        pp.scr = scr;
        pp.dev_err = dev_err;
        ScanParams sp;
        sp.L = L;
        sp.H = cfg_.H;
        sp.NC = NC;
        sp.gates = gates;
        sp.out_mode = mode;
        sp.acc = acc;
        sp.out = static_cast<__nv_bfloat16 *>(out);
        sp.dev_err = dev_err;
        CUtensorMap mout;
        sp.out_tma = scan_out_tma(&mout, mode, acc, out, cfg_.H, L, cfg_.B);
        int nlaunch = 0;
        for (int g = 0; g < segs && e == cudaSuccess; ++g) {
            const int c0 = g * per, n = min(per, NC - c0);
            if (n <= 0) break;
            const bool last = c0 + n >= NC;
            pp.c_begin = c0;
            gdn_prep_kernel<<<dim3(n, cfg_.H, cfg_.B), 128, prep_smem, prep_stream_>>>(mq, mk, mv, pp);
            e = cudaGetLastError();
            if (e == cudaSuccess) e = cudaEventRecord(ev_[1 + g], prep_stream_);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_[1 + g], 0);
            sp.c_begin = c0;
            sp.nseg = n;
            sp.S_in = g == 0 ? S_in : s_mid_ + (g & 1) * sstride;
            sp.S_out = last ? S_out : s_mid_ + ((g + 1) & 1) * sstride;
            if (e == cudaSuccess)
                gdn_scan_kernel<<<dim3(cfg_.H, cfg_.B), kScanThreads, scan_smem, s>>>(mwq, mk16, mpm, mut, mell,
                                                                                       mout, sp);
            if (e == cudaSuccess) e = cudaGetLastError();
            nlaunch += 2;
            if (last) break;
        }
        if (e != cudaSuccess) return e;
        *done = true;
        if (launches) *launches = nlaunch;
        return cudaGetLastError();
    }

private:
    hlta_config cfg_;
    static constexpr int kSegs = 4;
    int max_nc_;
    void *base_ = nullptr;
    float *s_mid_ = nullptr;
    cudaStream_t prep_stream_ = nullptr;
    cudaEvent_t ev_[1 + kSegs] = {};
    size_t bytes_ = 0;
    bool attr_set_ = false;
};

}  // namespace

TcGdn *TcGdn::create(const hlta_config &cfg, long long max_seq_len) {
    if (cfg.dtype != HLTA_BF16 || cfg.d_k != kD || cfg.d_v != kD) return nullptr;
    long long L = max_seq_len > cfg.max_stream_tokens ? max_seq_len : cfg.max_stream_tokens;
    const int max_nc = (int)((L + kC - 1) / kC);
    TcGdnImpl *g = new TcGdnImpl(cfg, max_nc);
    if (!g->init()) {
        delete g;
        return nullptr;
    }
    return g;
}

}  // namespace hlta

// =====================================================================
// hlta_gdn_forward_noalloc: the chunked memory branch without any device
// allocation.  Some callers may not allocate device memory once they are
// running -- for example a control loop under a fixed memory budget that
// reserves everything at start-up, or code inside a foreign allocator that
// forbids cudaMalloc.  They cannot create a handle (hlta_create allocates), so
// this entry point takes every size as an argument and runs the same prep and
// scan kernels on a scratch that lives in a file-scope __device__ array.
//
// The array is part of the library image: every GPU that loads the library
// holds its 96 MiB until the process exits.  All calls share it and it keeps
// the previous call's contents; each call clears what must start at zero (the
// device error word).  Calls whose executions overlap on the GPU (for example
// on two streams) race on it and must be ordered by the caller.
// =====================================================================
#include <mutex>

#include "hlta.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 96ull << 20;
// 256-byte aligned; the error word sits in the first 256 bytes, the chunk
// scratch starts at byte 256 (TMA needs 16-byte aligned bases, kept here).
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_base[kNoAllocMaxDevices];  // device address of the array, per device

constexpr size_t kNoAllocChunkBytes = hlta::kWQBytes + hlta::kK16Bytes + hlta::kPmBytes + hlta::kUtBytes +
                                      hlta::kEllBytes;

hlta_status noalloc_fail(hlta_status st, const char *msg) {
    hlta::set_last_error(msg);
    return st;
}

}  // namespace

extern "C" HLTA_API hlta_status hlta_gdn_forward_noalloc(int B, int L, int H, const void *q, const void *k,
                                                         const void *v, const float *alpha, const float *beta,
                                                         const float *gates, const float *S0, float *S_out,
                                                         void *out, void *stream) {
    using namespace hlta;
    if (B < 1 || H < 1 || L < kC)
        return noalloc_fail(HLTA_ERR_INVALID_ARG, "hlta_gdn_forward_noalloc: need B >= 1, H >= 1, L >= 64");
    const void *ptrs[] = {q, k, v, alpha, beta, gates, out};
    for (const void *ptr : ptrs)
        if (!ptr || (reinterpret_cast<uintptr_t>(ptr) & 15u))
            return noalloc_fail(HLTA_ERR_INVALID_ARG,
                                "hlta_gdn_forward_noalloc: a required pointer is NULL or not 16-byte aligned");
    if ((S0 && (reinterpret_cast<uintptr_t>(S0) & 15u)) || (S_out && (reinterpret_cast<uintptr_t>(S_out) & 15u)))
        return noalloc_fail(HLTA_ERR_INVALID_ARG, "hlta_gdn_forward_noalloc: S0/S_out not 16-byte aligned");
    const int NC = (L + kC - 1) / kC;
    const size_t n = (size_t)B * H * NC;
    if (256 + n * kNoAllocChunkBytes > kNoAllocScratchBytes)
        return noalloc_fail(HLTA_ERR_UNSUPPORTED,
                            "hlta_gdn_forward_noalloc: B*H*ceil(L/64) exceeds the 1110 chunk-heads of the "
                            "static 96 MiB scratch");

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
        return noalloc_fail(HLTA_ERR_CUDA, "hlta_gdn_forward_noalloc: no usable current device");
    char *base = nullptr;
    {
        // once per device, with that device current: the device address of the
        // array (the host-side symbol is not a device address) and the kernels'
        // shared-memory limits
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_base[dev]) {
            void *ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
                cudaGetLastError();
                return noalloc_fail(HLTA_ERR_CUDA, "hlta_gdn_forward_noalloc: cudaGetSymbolAddress failed");
            }
            if (cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(sizeof(PrepSmem) + 1024)) != cudaSuccess ||
                cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(sizeof(ScanSmem) + 1024)) != cudaSuccess) {
                cudaGetLastError();
                return noalloc_fail(HLTA_ERR_CUDA, "hlta_gdn_forward_noalloc: cudaFuncSetAttribute failed");
            }
            g_noalloc_base[dev] = ptr;
        }
        base = static_cast<char *>(g_noalloc_base[dev]);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int *dev_err = reinterpret_cast<int *>(base);
    GdnScratch scr;
    char *p = base + 256;
    scr.wq = reinterpret_cast<__half *>(p);
    p += n * kWQBytes;
    scr.k16 = reinterpret_cast<__half *>(p);
    p += n * kK16Bytes;
    scr.pm = reinterpret_cast<__half *>(p);
    p += n * kPmBytes;
    scr.ut = reinterpret_cast<float *>(p);
    p += n * kUtBytes;
    scr.ell = reinterpret_cast<float *>(p);

    CUtensorMap mq, mk, mv, mwq, mk16, mpm, mut, mell;
    if (!map_tokens(&mq, q, H, L, B) || !map_tokens(&mk, k, H, L, B) || !map_tokens(&mv, v, H, L, B) ||
        !map_2d(&mwq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, scr.wq, kD, n * 128, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mk16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, scr.k16, kD, n * kC, 64, kC, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mpm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, scr.pm, kC, n * kC, 64, kC, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mut, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, scr.ut, kD, n * kC, kD, kC, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !map_2d(&mell, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, scr.ell, 2 * kC, n, 2 * kC, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
        return noalloc_fail(HLTA_ERR_CUDA, "hlta_gdn_forward_noalloc: tensor map encoding failed");

    if (cudaMemsetAsync(dev_err, 0, sizeof(int), s) != cudaSuccess) {
        cudaGetLastError();
        return noalloc_fail(HLTA_ERR_CUDA, "hlta_gdn_forward_noalloc: clearing the error word failed");
    }
    PrepParams pp;
    pp.alpha = alpha;
    pp.beta = beta;
    pp.L = L;
    pp.H = H;
    pp.NC = NC;
    pp.c_begin = 0;
    pp.form = HLTA_GDN_DECAYED;
    pp.scr = scr;
    pp.dev_err = dev_err;
    gdn_prep_kernel<<<dim3(NC, H, B), 128, sizeof(PrepSmem) + 1024, s>>>(mq, mk, mv, pp);
    ScanParams sp;
    sp.L = L;
    sp.H = H;
    sp.NC = NC;
    sp.c_begin = 0;
    sp.nseg = NC;
    sp.S_in = S0;
    sp.S_out = S_out;
    sp.gates = gates;
    sp.out_mode = OUT_FINAL_ONLY;
    sp.acc = nullptr;
    sp.out = static_cast<__nv_bfloat16 *>(out);
    sp.dev_err = dev_err;
    CUtensorMap mout;
    sp.out_tma = scan_out_tma(&mout, OUT_FINAL_ONLY, nullptr, out, H, L, B);
    gdn_scan_kernel<<<dim3(H, B), kScanThreads, sizeof(ScanSmem) + 1024, s>>>(mwq, mk16, mpm, mut, mell, mout, sp);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return noalloc_fail(HLTA_ERR_CUDA, cudaGetErrorString(e));
    hlta::set_last_error("");
    return HLTA_OK;
}
