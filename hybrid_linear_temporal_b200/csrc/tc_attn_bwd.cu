// tc_attn_bwd.cu -- SWA / DSWA backward on the sm_100a tensor cores (bf16).
//
// Kairos paper, section 2.2.2 (Eq. (7) SWA, Eq. (8) DSWA): the gradient of the
// windowed softmax attention, with the segment geometry of the forward kernel
// (a segment is the whole sequence for SWA, one frame for DSWA; query r of a
// class attends to keys r - w < r_k <= r + w_hi).  With x = q.k log2(e)/sqrt(d),
// p = 2^(x - lse) (lse from the forward), dO = g dout (g the branch's gate),
// rd = dout . o:
//   dS = p (g dout.v - g rd)          (the 1/sqrt(d) of the logits is applied
//   dQ = dS K,  dK = dS^T Q,  dV = g P^T dout     to dQ and dK at the end)
// Two kernels, each one CTA per SM with 320 threads (warp 0 TMA, warp 1 TMEM
// allocation and the tcgen05.mma issue, warps 2-9 the elementwise work):
//   attn_bwd_dq_kernel   two 128-row query tiles per CTA, walking their key
//     tiles: S_j = Q_j K^T (SS) -> P in registers; dP_j = dO_j V^T (SS) into
//     the same TMEM columns once S_j is read; dS_j written back as bf16 over
//     them; dQ_j += dS_j K (TS form, K read MN-major).  TMEM: S/dP of tile 0
//     and 1 at columns 0-127 / 128-255, dQ_0 and dQ_1 at 256-383 / 384-511.
//   attn_bwd_dkv_kernel  one 128-key tile per CTA, walking the query tiles
//     whose window reaches it: S^T = K Q^T and dP^T = V dO^T (SS, keys on the
//     TMEM lanes), P^T and dS^T written back as bf16, dV += P^T dO and
//     dK += dS^T Q (TS form).  Warps 2-5 handle query columns 0-63, warps 6-9
//     columns 64-127, so each group writes its bf16 values over columns it
//     alone has read.  TMEM: S^T 0-127, dP^T 128-255, dV 256-383, dK 384-511.
// Tiles never straddle a segment; tiles crossing a band edge or a segment end
// are masked per element.  Every wait is bounded (sm100_ptx.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tc_attn_bwd.h"

namespace hlta {

namespace {

using namespace sm100;

constexpr int kT = 128;   // rows of a query tile and of a key tile
constexpr int kD = 128;   // head dim
constexpr int kMaxT = 40;
constexpr int kThreads = 320;
constexpr uint32_t kTileBytes = kT * kD * 2;     // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-column TMA box
constexpr int kSlotsQ = 3;                       // K/V ring of the dQ kernel
constexpr int kSlotsKV = 4;                      // Q/dO ring of the dK/dV kernel

struct Tile {
    int seg;    // segment row of the 4-D view: b*Fseg + f
    int s0;     // first row inside the segment
    int rbase;  // rearranged position of that row
    int valid;  // rows of this tile inside the segment
    uint8_t use[2], full[2];
};

struct BwdParams {
    int Pseg, Fseg, dil, w, w_hi, blocks_per_seg;
    int H, L;
    float scale_log2, scale;
    const float *gates;
    int gate_col;
    const float *lse, *rowdot;  // [B, H, L]
    float *dq, *dk, *dv;        // [B, L, H, 128] fp32, added to
    int *dev_err;
};

// Partner tiles (keys for the dQ kernel, queries for the dK/dV kernel) of the
// CTA's own tiles: own rows r in [r_min + 128 j, + nown[j]) reach partners r'
// with r - back < r' <= r + fwd, in the same class g.  Returns the count.
__device__ int build_tiles(Tile *out, const BwdParams &p, int b, int g, int r_min, const int (&nown)[2], int back,
                           int fwd) {
    int n = 0;
    const int r_max = r_min + nown[0] + nown[1] - 1;
    const int lo_r = r_min - back + 1, hi_r = r_max + fwd;
    const int m_last = (p.Fseg - 1 - g) / p.dil;
    for (int mm = min(m_last, hi_r / p.Pseg); mm >= 0; --mm) {
        const int base = mm * p.Pseg;
        if (base + p.Pseg - 1 < lo_r) break;
        const int s_lo = max(0, lo_r - base), s_hi = min(p.Pseg - 1, hi_r - base);
        for (int t = s_lo / kT; t <= s_hi / kT && n < kMaxT; ++t, ++n) {
            Tile &k = out[n];
            k.seg = b * p.Fseg + g + p.dil * mm;
            k.s0 = t * kT;
            k.rbase = base + t * kT;
            k.valid = min(kT, p.Pseg - t * kT);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int lo = r_min + j * kT, hi = lo + nown[j] - 1;
                k.use[j] = nown[j] > 0 && k.rbase <= hi + fwd && k.rbase + k.valid - 1 >= lo - back + 1;
                k.full[j] = k.valid == kT && k.rbase + kT - 1 <= lo + fwd && k.rbase > hi - back;
            }
        }
    }
    return n;
}

// 128x128x128 SS product: D = A B^T, A and B K-major 128-row tiles (two
// 64-column swizzled boxes each).
__device__ __forceinline__ void mma_ss_tile(uint32_t d_tmem, uint32_t a, uint32_t b, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk < 4) ? kk * 32 : kHalfBytes + (kk - 4) * 32;
        umma_ss(d_tmem, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), idesc,
                kk > 0 ? 1u : 0u);
    }
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
struct __align__(16) SmemQ {
    uint8_t q[2][kTileBytes];
    uint8_t dout[2][kTileBytes];
    uint8_t kv[kSlotsQ][kTileBytes];
    uint64_t bar_q, full[kSlotsQ], empty[kSlotsQ], bar_s[2], bar_sfree[2], bar_dp[2], bar_ds[2], bar_o;
    uint32_t tmem_base;
    int abort;
    int nkt;
    Tile kt[kMaxT];
};
static_assert(sizeof(SmemQ) + 1024 <= 232448, "dQ kernel shared memory exceeds 227 KB");

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    SmemQ &sm = *reinterpret_cast<SmemQ *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg_f = blockIdx.x / p.blocks_per_seg, qb = blockIdx.x % p.blocks_per_seg;
    const int h = blockIdx.y, b = blockIdx.z;
    const int s0 = qb * 2 * kT;
    const int nq0 = min(kT, p.Pseg - s0);
    const int nq1 = max(0, min(kT, p.Pseg - s0 - kT));
    const int g = seg_f % p.dil, m = seg_f / p.dil;
    const int r_min = m * p.Pseg + s0;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        const int nown[2] = {nq0, nq1};
        sm.nkt = build_tiles(sm.kt, p, b, g, r_min, nown, p.w, p.w_hi);
        sm.abort = *reinterpret_cast<volatile int *>(p.dev_err) != 0 ? 1 : 0;
        mbar_init(&sm.bar_q, 1);
        for (int i = 0; i < kSlotsQ; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sm.bar_s[j], 1);
            mbar_init(&sm.bar_sfree[j], 128);
            mbar_init(&sm.bar_dp[j], 1);
            mbar_init(&sm.bar_ds[j], 128);
        }
        mbar_init(&sm.bar_o, 1);
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
    const int nkt = sm.nkt;
    const int nqt = nq1 > 0 ? 2 : 1;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && !*abort) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            prefetch_tensormap(&tmO);
            const int qseg = b * p.Fseg + seg_f;
            mbar_expect_tx(&sm.bar_q, 2 * nqt * kTileBytes);
            for (int j = 0; j < nqt; ++j) {
                tma_load_4d(sm.q[j], &tmQ, 0, h, s0 + j * kT, qseg, &sm.bar_q);
                tma_load_4d(sm.q[j] + kHalfBytes, &tmQ, 64, h, s0 + j * kT, qseg, &sm.bar_q);
                tma_load_4d(sm.dout[j], &tmO, 0, h, s0 + j * kT, qseg, &sm.bar_q);
                tma_load_4d(sm.dout[j] + kHalfBytes, &tmO, 64, h, s0 + j * kT, qseg, &sm.bar_q);
            }
            int issued = 0;
            for (int u = 0; u < 2 * nkt; ++u) {
                const int slot = u % kSlotsQ;
                if (u >= kSlotsQ && !mbar_wait(&sm.empty[slot], ((u / kSlotsQ) - 1) & 1, abort, p.dev_err)) break;
                const Tile &kt = sm.kt[u >> 1];
                const CUtensorMap *map = (u & 1) ? &tmV : &tmK;
                mbar_expect_tx(&sm.full[slot], kTileBytes);
                tma_load_4d(sm.kv[slot], map, 0, h, kt.s0, kt.seg, &sm.full[slot]);
                tma_load_4d(sm.kv[slot] + kHalfBytes, map, 64, h, kt.s0, kt.seg, &sm.full[slot]);
                issued = u + 1;
            }
            if (*abort) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                mbar_wait(&sm.bar_q, 0, no_abort, nullptr);
                for (int u = (issued > kSlotsQ ? issued - kSlotsQ : 0); u < issued; ++u)
                    mbar_wait(&sm.full[u % kSlotsQ], (u / kSlotsQ) & 1, no_abort, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // Key tile t: dP_0(t), dP_1(t) once each S_j(t) is read; then dQ_j(t)
        // once dS_j(t) is written, followed by S_j(t+1) over the same columns.
        if (lane == 0) {
            const uint32_t idesc_ss = idesc_bf16_f32(128, 128, 0, 0);
            const uint32_t idesc_ts = idesc_bf16_f32(128, 128, 0, 1);
            int ns[2] = {0, 0};
            bool live = !*abort && mbar_wait(&sm.bar_q, 0, abort, p.dev_err);
            if (live && nkt > 0) {
                live = mbar_wait(&sm.full[0], 0, abort, p.dev_err);
                if (live) {
                    tc_fence_after();
                    for (int j = 0; j < 2; ++j)
                        if (sm.kt[0].use[j]) {
                            mma_ss_tile(tmem + j * 128, smem_u32(sm.q[j]), smem_u32(sm.kv[0]), idesc_ss);
                            umma_commit(&sm.bar_s[j]);
                        }
                }
            }
            for (int t = 0; t < nkt && live; ++t) {
                const Tile kt = sm.kt[t];
                const int uk = 2 * t, sk = uk % kSlotsQ, uv = 2 * t + 1, sv = uv % kSlotsQ;
                if (!(live = mbar_wait(&sm.full[sv], (uv / kSlotsQ) & 1, abort, p.dev_err))) break;
                for (int j = 0; j < 2 && live; ++j) {
                    if (!kt.use[j]) continue;
                    if (!(live = mbar_wait(&sm.bar_sfree[j], ns[j] & 1, abort, p.dev_err))) break;
                    tc_fence_after();
                    mma_ss_tile(tmem + j * 128, smem_u32(sm.dout[j]), smem_u32(sm.kv[sv]), idesc_ss);
                    umma_commit(&sm.bar_dp[j]);
                }
                if (!live) break;
                umma_commit(&sm.empty[sv]);
                const bool more = t + 1 < nkt;
                const int uk2 = 2 * (t + 1), sk2 = uk2 % kSlotsQ;
                bool k2_ready = false;
                const uint32_t ka = smem_u32(sm.kv[sk]);
                for (int j = 0; j < 2 && live; ++j) {
                    if (kt.use[j]) {
                        if (!(live = mbar_wait(&sm.bar_ds[j], ns[j] & 1, abort, p.dev_err))) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < kT / 16; ++kk)
                            umma_ts(tmem + 256 + j * 128, tmem + j * 128 + kk * 8,
                                    smem_desc_sw128(ka + kk * 2048, kHalfBytes, 1024), idesc_ts,
                                    (ns[j] > 0 || kk > 0) ? 1u : 0u);
                        ++ns[j];
                    }
                    if (more && sm.kt[t + 1].use[j]) {
                        if (!k2_ready) {
                            if (!(live = mbar_wait(&sm.full[sk2], (uk2 / kSlotsQ) & 1, abort, p.dev_err))) break;
                            k2_ready = true;
                        }
                        tc_fence_after();
                        mma_ss_tile(tmem + j * 128, smem_u32(sm.q[j]), smem_u32(sm.kv[sk2]), idesc_ss);
                        umma_commit(&sm.bar_s[j]);
                    }
                }
                if (!live) break;
                umma_commit(&sm.empty[sk]);
                if (more && !k2_ready && !(live = mbar_wait(&sm.full[sk2], (uk2 / kSlotsQ) & 1, abort, p.dev_err)))
                    break;
            }
            umma_commit(&sm.bar_o);
            if (*abort) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                mbar_wait(&sm.bar_o, 0, no_abort, nullptr);
            }
        }
    } else {
        // ------------------------------------------------ P, dS and the dQ epilogue of tile j
        const int j = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t colR = j * 128, colQ = 256 + j * 128;
        const int nqj = j == 0 ? nq0 : nq1;
        const int r_q = r_min + j * kT + row;
        const int tok = seg_f * p.Pseg + s0 + j * kT + row;
        const size_t hm = ((size_t)b * p.H + h) * p.L + tok;
        const float lse = row < nqj ? p.lse[hm] : 0.f;
        const float gt = p.gates[h * 3 + p.gate_col];
        const float grd = row < nqj ? gt * p.rowdot[hm] : 0.f;
        const float sl2 = p.scale_log2;
        int n = 0;
        bool ok = !*abort && nqj > 0;
        for (int t = 0; t < nkt && ok; ++t) {
            const Tile &ktr = sm.kt[t];
            if (!ktr.use[j]) continue;
            const bool full = ktr.full[j];
            const int rbase = ktr.rbase, kvalid = ktr.valid;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_s[j], n & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s[128];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tmem_ld32(tl + colR + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * i]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_sfree[j]);
            const int lo = full ? 0 : max(0, r_q - p.w + 1 - rbase);
            const int hi = full ? kT - 1 : min(kvalid - 1, r_q + p.w_hi - rbase);
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                const float x = ex2(fmaf(__uint_as_float(s[c]), sl2, -lse));
                s[c] = __float_as_uint(c >= lo && c <= hi ? x : 0.f);
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_dp[j], n & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t d[32];
                tmem_ld32(tl + colR + 32 * c4, d);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float a0 = __uint_as_float(s[32 * c4 + 2 * e]);
                    const float a1 = __uint_as_float(s[32 * c4 + 2 * e + 1]);
                    pk[e] = pack_bf16x2(a0 * fmaf(gt, __uint_as_float(d[2 * e]), -grd),
                                        a1 * fmaf(gt, __uint_as_float(d[2 * e + 1]), -grd));
                }
                tmem_st16(tl + colR + 16 * c4, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_ds[j]);
            ++n;
        }
        if (ok && n > 0 && __all_sync(0xffffffffu, mbar_wait(&sm.bar_o, 0, abort, p.dev_err))) {
            tc_fence_after();
            float *dqp = p.dq + (((size_t)b * p.L + tok) * p.H + h) * kD;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t r[32];
                tmem_ld32(tl + colQ + 32 * c4, r);
                tmem_wait_ld();
                if (row < nqj) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        float4 v = *reinterpret_cast<float4 *>(dqp + 32 * c4 + e);
                        v.x = fmaf(__uint_as_float(r[e]), p.scale, v.x);
                        v.y = fmaf(__uint_as_float(r[e + 1]), p.scale, v.y);
                        v.z = fmaf(__uint_as_float(r[e + 2]), p.scale, v.z);
                        v.w = fmaf(__uint_as_float(r[e + 3]), p.scale, v.w);
                        *reinterpret_cast<float4 *>(dqp + 32 * c4 + e) = v;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
struct __align__(16) SmemKV {
    uint8_t k[kTileBytes];
    uint8_t v[kTileBytes];
    uint8_t qd[kSlotsKV][kTileBytes];
    float lse[2][kT], rd[2][kT];
    uint64_t bar_kv, full[kSlotsKV], empty[kSlotsKV], bar_s, bar_dp, bar_p, bar_ds, bar_o, bar_ld[2];
    uint32_t tmem_base;
    int abort;
    int nqt;
    Tile qt[kMaxT];
};
static_assert(sizeof(SmemKV) + 1024 <= 232448, "dK/dV kernel shared memory exceeds 227 KB");

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    SmemKV &sm = *reinterpret_cast<SmemKV *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg_f = blockIdx.x / p.blocks_per_seg, kb = blockIdx.x % p.blocks_per_seg;
    const int h = blockIdx.y, b = blockIdx.z;
    const int s0 = kb * kT;
    const int kvalid = min(kT, p.Pseg - s0);
    const int g = seg_f % p.dil, m = seg_f / p.dil;
    const int r_min = m * p.Pseg + s0;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        // queries reaching key r_k: r_k - w_hi <= r_q <= r_k + w - 1
        const int nown[2] = {kvalid, 0};
        sm.nqt = build_tiles(sm.qt, p, b, g, r_min, nown, p.w_hi + 1, p.w - 1);
        sm.abort = *reinterpret_cast<volatile int *>(p.dev_err) != 0 ? 1 : 0;
        mbar_init(&sm.bar_kv, 1);
        for (int i = 0; i < kSlotsKV; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        mbar_init(&sm.bar_s, 1);
        mbar_init(&sm.bar_dp, 1);
        mbar_init(&sm.bar_p, 256);
        mbar_init(&sm.bar_ds, 256);
        mbar_init(&sm.bar_o, 1);
        mbar_init(&sm.bar_ld[0], 256);
        mbar_init(&sm.bar_ld[1], 256);
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
    const int nqt = sm.nqt;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && !*abort) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            prefetch_tensormap(&tmO);
            const int kseg = b * p.Fseg + seg_f;
            mbar_expect_tx(&sm.bar_kv, 2 * kTileBytes);
            tma_load_4d(sm.k, &tmK, 0, h, s0, kseg, &sm.bar_kv);
            tma_load_4d(sm.k + kHalfBytes, &tmK, 64, h, s0, kseg, &sm.bar_kv);
            tma_load_4d(sm.v, &tmV, 0, h, s0, kseg, &sm.bar_kv);
            tma_load_4d(sm.v + kHalfBytes, &tmV, 64, h, s0, kseg, &sm.bar_kv);
            int issued = 0;
            for (int u = 0; u < 2 * nqt; ++u) {
                const int slot = u % kSlotsKV;
                if (u >= kSlotsKV && !mbar_wait(&sm.empty[slot], ((u / kSlotsKV) - 1) & 1, abort, p.dev_err)) break;
                const Tile &qt = sm.qt[u >> 1];
                const CUtensorMap *map = (u & 1) ? &tmO : &tmQ;
                mbar_expect_tx(&sm.full[slot], kTileBytes);
                tma_load_4d(sm.qd[slot], map, 0, h, qt.s0, qt.seg, &sm.full[slot]);
                tma_load_4d(sm.qd[slot] + kHalfBytes, map, 64, h, qt.s0, qt.seg, &sm.full[slot]);
                issued = u + 1;
            }
            if (*abort) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                mbar_wait(&sm.bar_kv, 0, no_abort, nullptr);
                for (int u = (issued > kSlotsKV ? issued - kSlotsKV : 0); u < issued; ++u)
                    mbar_wait(&sm.full[u % kSlotsKV], (u / kSlotsKV) & 1, no_abort, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // Query tile i: dV += P^T(i) dO_i, then S^T(i+1); dK += dS^T(i) Q_i, then
        // dP^T(i+1).  S^T(i+1) and dP^T(i+1) overwrite the columns those TS
        // products read, after them in this thread's issue order.
        if (lane == 0) {
            const uint32_t idesc_ss = idesc_bf16_f32(128, 128, 0, 0);
            const uint32_t idesc_ts = idesc_bf16_f32(128, 128, 0, 1);
            const uint32_t ka = smem_u32(sm.k), va = smem_u32(sm.v);
            // P^T / dS^T of query columns 64G.. are at TMEM columns 64G .. 64G+31
            auto acol = [](int kk) { return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8); };
            bool live = !*abort && mbar_wait(&sm.bar_kv, 0, abort, p.dev_err);
            if (live && nqt > 0) {
                live = mbar_wait(&sm.full[0], 0, abort, p.dev_err);
                if (live) {
                    tc_fence_after();
                    mma_ss_tile(tmem, ka, smem_u32(sm.qd[0]), idesc_ss);
                    umma_commit(&sm.bar_s);
                    live = mbar_wait(&sm.full[1], 0, abort, p.dev_err);
                }
                if (live) {
                    tc_fence_after();
                    mma_ss_tile(tmem + 128, va, smem_u32(sm.qd[1]), idesc_ss);
                    umma_commit(&sm.bar_dp);
                }
            }
            for (int i = 0; i < nqt && live; ++i) {
                const int sq = (2 * i) % kSlotsKV, so = (2 * i + 1) % kSlotsKV;
                const bool more = i + 1 < nqt;
                const int uq2 = 2 * i + 2, uo2 = 2 * i + 3;
                if (!(live = mbar_wait(&sm.bar_p, i & 1, abort, p.dev_err))) break;
                tc_fence_after();
                const uint32_t oa = smem_u32(sm.qd[so]);
#pragma unroll
                for (int kk = 0; kk < kT / 16; ++kk)
                    umma_ts(tmem + 256, tmem + acol(kk), smem_desc_sw128(oa + kk * 2048, kHalfBytes, 1024), idesc_ts,
                            (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.empty[so]);
                if (more) {
                    if (!(live = mbar_wait(&sm.full[uq2 % kSlotsKV], (uq2 / kSlotsKV) & 1, abort, p.dev_err))) break;
                    tc_fence_after();
                    mma_ss_tile(tmem, ka, smem_u32(sm.qd[uq2 % kSlotsKV]), idesc_ss);
                    umma_commit(&sm.bar_s);
                }
                if (!(live = mbar_wait(&sm.bar_ds, i & 1, abort, p.dev_err))) break;
                tc_fence_after();
                const uint32_t qa = smem_u32(sm.qd[sq]);
#pragma unroll
                for (int kk = 0; kk < kT / 16; ++kk)
                    umma_ts(tmem + 384, tmem + 128 + acol(kk), smem_desc_sw128(qa + kk * 2048, kHalfBytes, 1024),
                            idesc_ts, (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.empty[sq]);
                if (more) {
                    if (!(live = mbar_wait(&sm.full[uo2 % kSlotsKV], (uo2 / kSlotsKV) & 1, abort, p.dev_err))) break;
                    tc_fence_after();
                    mma_ss_tile(tmem + 128, va, smem_u32(sm.qd[uo2 % kSlotsKV]), idesc_ss);
                    umma_commit(&sm.bar_dp);
                }
            }
            umma_commit(&sm.bar_o);
            if (*abort) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                mbar_wait(&sm.bar_o, 0, no_abort, nullptr);
            }
        }
    } else {
        // ------------------------------------------------ P^T, dS^T and the dK/dV epilogue
        const int G = (warp - 2) >> 2;  // query columns 64G .. 64G+63
        const int quad = warp & 3;
        const int row = quad * 32 + lane;  // key row = TMEM lane
        const int tt = G * kT + row;       // loader index 0..255
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const int r_k = r_min + row;
        const float gt = p.gates[h * 3 + p.gate_col];
        const float sl2 = p.scale_log2;
        const size_t hm0 = ((size_t)b * p.H + h) * p.L;
        bool ok = !*abort;
        int n = 0;
        for (int i = 0; i < nqt && ok; ++i) {
            const Tile &qt = sm.qt[i];
            const int buf = i & 1;
            {
                const int c = tt & (kT - 1);
                const int tok = (qt.seg - b * p.Fseg) * p.Pseg + qt.s0 + c;
                const bool valid = c < qt.valid;
                if (tt < kT)
                    sm.lse[buf][c] = valid ? p.lse[hm0 + tok] : 0.f;
                else
                    sm.rd[buf][c] = valid ? p.rowdot[hm0 + tok] : 0.f;
            }
            // every loader has written this tile's values (and so has finished
            // reading the buffer's previous tile, two iterations back)
            mbar_arrive(&sm.bar_ld[buf]);
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_ld[buf], (i >> 1) & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            const int lo = qt.full[0] ? 0 : max(0, r_k - p.w_hi - qt.rbase);
            const int hi = qt.full[0] ? kT - 1 : min(qt.valid - 1, r_k + p.w - 1 - qt.rbase);
            const int lo_g = row < kvalid ? lo - 64 * G : 64, hi_g = hi - 64 * G;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_s, i & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s[64];
            tmem_ld32(tl + 64 * G, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
            tmem_ld32(tl + 64 * G + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float x = ex2(fmaf(__uint_as_float(s[c]), sl2, -sm.lse[buf][64 * G + c]));
                s[c] = __float_as_uint(c >= lo_g && c <= hi_g ? x : 0.f);
            }
            {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1]));
                tmem_st32(tl + 64 * G, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_p);
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_dp, i & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                uint32_t d[32];
                tmem_ld32(tl + 128 + 64 * G + 32 * c2, d);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c = 32 * c2 + 2 * e;
                    const float r0 = sm.rd[buf][64 * G + c], r1 = sm.rd[buf][64 * G + c + 1];
                    pk[e] = pack_bf16x2(__uint_as_float(s[c]) * gt * (__uint_as_float(d[2 * e]) - r0),
                                        __uint_as_float(s[c + 1]) * gt * (__uint_as_float(d[2 * e + 1]) - r1));
                }
                tmem_st16(tl + 128 + 64 * G + 16 * c2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_ds);
            ++n;
        }
        if (ok && n > 0 && __all_sync(0xffffffffu, mbar_wait(&sm.bar_o, 0, abort, p.dev_err))) {
            tc_fence_after();
            const int ktok = seg_f * p.Pseg + s0 + row;
            const size_t o = (((size_t)b * p.L + ktok) * p.H + h) * kD + 64 * G;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                uint32_t rv[32], rk[32];
                tmem_ld32(tl + 256 + 64 * G + 32 * c2, rv);
                tmem_ld32(tl + 384 + 64 * G + 32 * c2, rk);
                tmem_wait_ld();
                if (row < kvalid) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        float4 a = *reinterpret_cast<float4 *>(p.dv + o + 32 * c2 + e);
                        a.x = fmaf(__uint_as_float(rv[e]), gt, a.x);
                        a.y = fmaf(__uint_as_float(rv[e + 1]), gt, a.y);
                        a.z = fmaf(__uint_as_float(rv[e + 2]), gt, a.z);
                        a.w = fmaf(__uint_as_float(rv[e + 3]), gt, a.w);
                        *reinterpret_cast<float4 *>(p.dv + o + 32 * c2 + e) = a;
                        float4 c = *reinterpret_cast<float4 *>(p.dk + o + 32 * c2 + e);
                        c.x = fmaf(__uint_as_float(rk[e]), p.scale, c.x);
                        c.y = fmaf(__uint_as_float(rk[e + 1]), p.scale, c.y);
                        c.z = fmaf(__uint_as_float(rk[e + 2]), p.scale, c.z);
                        c.w = fmaf(__uint_as_float(rk[e + 3]), p.scale, c.w);
                        *reinterpret_cast<float4 *>(p.dk + o + 32 * c2 + e) = c;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side
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

// 4-D view (d, H, Pseg, B*Fseg) of a [B, L, H, 128] bf16 tensor, box (64, 1, 128, 1).
bool make_map(CUtensorMap *map, const void *base, int H, int Pseg, int segs) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)Pseg, (cuuint64_t)segs};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)Pseg * H * kD * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kT, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

class TcAttnBwdImpl : public TcAttnBwd {
public:
    explicit TcAttnBwdImpl(const hlta_config &c) : cfg_(c) {}

    // The forward kernel's segment geometry (same coverage rule).
    static bool geometry(int L, WindowGeom g, int *Pseg, int *Fseg) {
        if (g.dil == 1) {
            *Pseg = L;
            *Fseg = 1;
        } else {
            if (L % g.P != 0) return false;
            *Pseg = g.P;
            *Fseg = L / g.P;
        }
        if (*Pseg < kT) return false;
        const long long span = (long long)g.w + g.w_hi + 2 * kT - 1;
        const long long bound = (span + kT - 1) / kT + 2 * (span / *Pseg + 2);
        if (bound > kMaxT) return false;
        return (long long)*Fseg * *Pseg <= (1LL << 30);
    }

    bool covers(int L, WindowGeom g) const override {
        int a, b;
        return geometry(L, g, &a, &b);
    }

    cudaError_t run(const void *q, const void *k, const void *v, const void *dout, int L, WindowGeom g,
                    const float *gates, int gate_col, const float *lse, const float *rowdot, float *dq, float *dk,
                    float *dv, int *dev_err, cudaStream_t s) override {
        int Pseg, Fseg;
        if (!geometry(L, g, &Pseg, &Fseg)) return cudaErrorInvalidValue;
        CUtensorMap mq, mk, mv, mo;
        const int segs = cfg_.B * Fseg;
        if (!make_map(&mq, q, cfg_.H, Pseg, segs) || !make_map(&mk, k, cfg_.H, Pseg, segs) ||
            !make_map(&mv, v, cfg_.H, Pseg, segs) || !make_map(&mo, dout, cfg_.H, Pseg, segs))
            return cudaErrorInvalidValue;
        BwdParams p;
        p.Pseg = Pseg;
        p.Fseg = Fseg;
        p.dil = g.dil;
        p.w = g.w;
        p.w_hi = g.w_hi;
        p.H = cfg_.H;
        p.L = L;
        p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
        p.scale = 1.f / sqrtf((float)kD);
        p.gates = gates;
        p.gate_col = gate_col;
        p.lse = lse;
        p.rowdot = rowdot;
        p.dq = dq;
        p.dk = dk;
        p.dv = dv;
        p.dev_err = dev_err;
        const size_t smq = sizeof(SmemQ) + 1024, smkv = sizeof(SmemKV) + 1024;
        if (!attr_set_) {
            cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smq);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(attn_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smkv);
            if (e != cudaSuccess) return e;
            attr_set_ = true;
        }
        p.blocks_per_seg = (Pseg + 2 * kT - 1) / (2 * kT);
        attn_bwd_dq_kernel<<<dim3(Fseg * p.blocks_per_seg, cfg_.H, cfg_.B), kThreads, smq, s>>>(mq, mk, mv, mo, p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        p.blocks_per_seg = (Pseg + kT - 1) / kT;
        attn_bwd_dkv_kernel<<<dim3(Fseg * p.blocks_per_seg, cfg_.H, cfg_.B), kThreads, smkv, s>>>(mq, mk, mv, mo,
                                                                                                   p);
        return cudaGetLastError();
    }

private:
    hlta_config cfg_;
    bool attr_set_ = false;
};

}  // namespace

TcAttnBwd *TcAttnBwd::create(const hlta_config &cfg) {
    if (cfg.dtype != HLTA_BF16 || cfg.d_k != kD || cfg.d_v != kD) return nullptr;
    return new TcAttnBwdImpl(cfg);
}

}  // namespace hlta
