// tc_attention.cu -- SWA / DSWA forward on the sm_100a tensor cores (bf16).
//
// Kairos paper, section 2.2.2: SWA (Eq. (7), causal window of w keys) and DSWA
// (Eq. (8): SWA after rearranging frames into residue classes f mod d).
//
// Both branches run as one kernel over "segments".  A segment is a run of
// Pseg consecutive tokens of one (batch, head) sequence: the whole sequence for
// SWA (Pseg = L), one latent frame for DSWA (Pseg = P).  Segment f of a batch
// belongs to class g = f mod dil at class position m = f / dil; a token s of it
// sits at rearranged position r = m*Pseg + s, and query r attends to the keys of
// its class with r - w < r_k <= r + w_hi (w_hi = 0: the causal window; w_hi > 0:
// the centred window Eq. (7) prints).  SWA is dil = 1 with one segment.  No
// rearranged copy is made: TMA reads tiles straight from the caller's
// [B, L, H, d] tensors through a 4-D view (d, H, Pseg, B*F), whose
// out-of-range rows arrive as zeros.
//
// One CTA (one per SM) handles two adjacent 128-row query tiles of a segment,
// which share every K/V tile:
//   warp 0      TMA producer: Q0, Q1, then K_t and V_t through a 5-slot ring
//   warp 1      TMEM allocation (512 columns); lane 0 issues tcgen05.mma
//                 S_j = Q_j K_t^T   (SS form, 128x128x128, fp32 in TMEM)
//                 O_j += P_j V_t    (TS form: P_j read from TMEM, V_t MN-major)
//               in the order PV0(t), QK0(t+1), PV1(t), QK1(t+1), so that the
//               softmax of one query tile runs under the other tile's MMAs
//   warps 2-5   softmax of tile 0, warps 6-9 softmax of tile 1: thread = query
//               row = TMEM lane.  Each row of S_j is read from TMEM once; online
//               softmax in the log2 domain with a lazily moved reference maximum
//               (O_j is rescaled in TMEM only when a row maximum grows by more
//               than 2^8); P_j is written back as bf16 over the first 64 columns
//               of S_j; the epilogue scales O_j by gate/l and writes rows.
// TMEM: S0/P0 cols 0-127, S1/P1 128-255, O0 256-383, O1 384-511.
// P_j aliases S_j: QK_j(t+1) is issued after PV_j(t) by the same thread, and
// the tensor pipe executes one thread's MMAs in issue order, so PV_j(t) has read
// P_j before QK_j(t+1) overwrites it.  For the same reason the commit that
// signals S_j(t) also covers PV_j(t-1): the softmax may rescale O_j as soon as
// S_j(t) is ready.
// Key tiles never straddle a segment; a tile is skipped for a query tile whose
// band it misses, and tiles crossing a band edge or a segment end are masked
// per element.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdio.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tc_attention.h"

namespace hlta {

namespace {

using namespace sm100;

constexpr int kBM = 128;   // rows per query tile
constexpr int kQT = 2;     // query tiles per CTA
constexpr int kBN = 128;   // keys per tile
constexpr int kD = 128;    // head dim (d_k = d_v)
constexpr int kMaxKT = 40;
constexpr int kThreads = 320;
constexpr int kSlots = 5;                        // K/V ring slots (one 128x128 bf16 tile each)
constexpr uint32_t kTileBytes = kBN * kD * 2;    // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-column TMA box
constexpr float kRescaleThreshold = 8.0f;        // log2 units

struct KeyTile {
    int seg;     // segment row of the 4-D view: b*Fseg + f
    int s0;      // first key row inside the segment
    int rbase;   // rearranged position of that row
    int kvalid;  // rows of this tile inside the segment
    float sk;    // FP8 variant: the e4m3 scale of this k tile (1 otherwise)
    uint8_t use[kQT], full[kQT];
};

struct TcAttnParams {
    int Pseg, Fseg, dil, w, w_hi, qblocks_per_seg;
    int H, L;
    float scale_log2;
    const float *gates;
    int gate_col, out_mode;
    float *acc;
    const float *acc2;  // optional second accumulator, added in the final modes
    __nv_bfloat16 *out;
    float *lse_out;  // optional [B, H, L]: log2-domain log-sum-exp of each row's scaled scores
    // FP8 variant: per-tile scales of the e4m3 q and k, [B*Fseg][H][nblk] (128-row blocks)
    const float *sq, *sk;
    int nblk;
    int *dev_err;
};

// 1024-byte aligned by the kernel (tiles first, each a multiple of 1 KB); the
// struct itself is not padded to 1 KB so that it fits the 227 KB limit.
struct __align__(16) Smem {
    uint8_t q[kQT][kTileBytes];
    uint8_t kv[kSlots][kTileBytes];
    uint64_t bar_q, full[kSlots], empty[kSlots], bar_s[kQT], bar_p[kQT], bar_o;
    uint32_t tmem_base;
    int abort;
    int nkt;
    KeyTile kt[kMaxKT];
};

static_assert(sizeof(Smem) + 1024 <= 232448, "attention shared memory exceeds the 227 KB per-block limit");

// Write 32 columns [c0, c0+32) of one output row with the OutMode semantics.
// The accumulator values are all loaded before any store, so the loads overlap
// instead of waiting on the stores before them.
__device__ __forceinline__ void store_chunk(const TcAttnParams &p, size_t base, int c0, const uint32_t (&o)[32],
                                            float scale) {
    float *__restrict__ acc = p.acc + base + c0;
    __nv_bfloat16 *__restrict__ out = p.out + base + c0;
    float a[32];
    if (p.out_mode == OUT_ADD || p.out_mode == OUT_FINAL) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(acc + c);
            a[c] = v.x;
            a[c + 1] = v.y;
            a[c + 2] = v.z;
            a[c + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) a[c] = 0.f;
    }
    if (p.acc2 && (p.out_mode == OUT_FINAL || p.out_mode == OUT_FINAL_ONLY)) {
        const float *__restrict__ acc2 = p.acc2 + base + c0;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(acc2 + c);
            a[c] += v.x;
            a[c + 1] += v.y;
            a[c + 2] += v.z;
            a[c + 3] += v.w;
        }
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) a[c] = fmaf(__uint_as_float(o[c]), scale, a[c]);
    if (p.out_mode == OUT_STORE || p.out_mode == OUT_ADD) {
#pragma unroll
        for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4 *>(acc + c) = make_float4(a[c], a[c + 1], a[c + 2], a[c + 3]);
    } else {
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
            uint4 w;
            w.x = pack_bf16x2(a[c], a[c + 1]);
            w.y = pack_bf16x2(a[c + 2], a[c + 3]);
            w.z = pack_bf16x2(a[c + 4], a[c + 5]);
            w.w = pack_bf16x2(a[c + 6], a[c + 7]);
            *reinterpret_cast<uint4 *>(out + c) = w;
        }
    }
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// kF8: q and k arrive as e4m3 tiles (128 one-byte columns, one TMA box) with a
// scale per 128-row tile; Q K^T runs as kind::f8f6f4 and the two tiles' scales
// multiply the softmax exponent.  P V stays bf16.
template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const TcAttnParams p) {
    constexpr uint32_t kQKBytes = kF8 ? kTileBytes / 2 : kTileBytes;  // one Q or K tile
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg_f = blockIdx.x / p.qblocks_per_seg;
    const int qb = blockIdx.x % p.qblocks_per_seg;
    const int h = blockIdx.y, b = blockIdx.z;
    const int s0 = qb * kQT * kBM;
    const int nq0 = min(kBM, p.Pseg - s0);
    const int nq1 = max(0, min(kBM, p.Pseg - s0 - kBM));
    const int g = seg_f % p.dil, m = seg_f / p.dil;
    const int r_min = m * p.Pseg + s0, r_max = r_min + nq0 + nq1 - 1;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        int n = 0;
        const int lo_r = r_min - p.w + 1, hi_r = r_max + p.w_hi;
        const int nqs[kQT] = {nq0, nq1};
        // class positions from the last one the forward reach touches down to the
        // first the backward reach touches
        const int m_last = (p.Fseg - 1 - g) / p.dil;
        for (int mm = min(m_last, hi_r / p.Pseg); mm >= 0; --mm) {
            const int base = mm * p.Pseg;
            if (base + p.Pseg - 1 < lo_r) break;
            const int s_lo = max(0, lo_r - base), s_hi = min(p.Pseg - 1, hi_r - base);
            for (int t = s_lo / kBN; t <= s_hi / kBN && n < kMaxKT; ++t, ++n) {
                KeyTile &k = sm.kt[n];
                k.seg = b * p.Fseg + g + p.dil * mm;
                k.s0 = t * kBN;
                k.rbase = base + t * kBN;
                k.kvalid = min(kBN, p.Pseg - t * kBN);
                k.sk = kF8 ? p.sk[((size_t)k.seg * p.H + h) * p.nblk + t] : 1.f;
#pragma unroll
                for (int j = 0; j < kQT; ++j) {
                    const int lo = r_min + j * kBM, hi = lo + nqs[j] - 1;
                    k.use[j] = nqs[j] > 0 && k.rbase <= hi + p.w_hi && k.rbase + k.kvalid - 1 >= lo - p.w + 1;
                    k.full[j] = k.kvalid == kBN && k.rbase + kBN - 1 <= lo + p.w_hi && k.rbase > hi - p.w;
                }
            }
        }
        sm.nkt = n;
        // an earlier launch gave up a wait: do no work (the error stays reported)
        sm.abort = *reinterpret_cast<volatile int *>(p.dev_err) != 0 ? 1 : 0;
        mbar_init(&sm.bar_q, 1);
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        for (int j = 0; j < kQT; ++j) {
            mbar_init(&sm.bar_s[j], 1);
            mbar_init(&sm.bar_p[j], 128);
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

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && !*abort) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            const int qseg = b * p.Fseg + seg_f;
            mbar_expect_tx(&sm.bar_q, nq1 > 0 ? 2 * kQKBytes : kQKBytes);
            for (int j = 0; j < (nq1 > 0 ? 2 : 1); ++j) {
                tma_load_4d(sm.q[j], &tmQ, 0, h, s0 + j * kBM, qseg, &sm.bar_q);
                if (!kF8) tma_load_4d(sm.q[j] + kHalfBytes, &tmQ, 64, h, s0 + j * kBM, qseg, &sm.bar_q);
            }
            int issued = 0;
            for (int u = 0; u < 2 * nkt; ++u) {
                const int slot = u % kSlots;
                if (u >= kSlots && !mbar_wait(&sm.empty[slot], ((u / kSlots) - 1) & 1, abort, p.dev_err)) break;
                const KeyTile &kt = sm.kt[u >> 1];
                const CUtensorMap *map = (u & 1) ? &tmV : &tmK;
                const bool one_box = kF8 && !(u & 1);
                mbar_expect_tx(&sm.full[slot], one_box ? kQKBytes : kTileBytes);
                tma_load_4d(sm.kv[slot], map, 0, h, kt.s0, kt.seg, &sm.full[slot]);
                if (!one_box) tma_load_4d(sm.kv[slot] + kHalfBytes, map, 64, h, kt.s0, kt.seg, &sm.full[slot]);
                issued = u + 1;
            }
            if (*abort) {
                // let copies in flight land before the CTA's shared memory is released
                int dummy = 0;
                volatile int *no_abort = &dummy;
                mbar_wait(&sm.bar_q, 0, no_abort, nullptr);
                for (int u = (issued > kSlots ? issued - kSlots : 0); u < issued; ++u)
                    mbar_wait(&sm.full[u % kSlots], (u / kSlots) & 1, no_abort, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // Per key tile t: PV0(t), QK0(t+1), PV1(t), QK1(t+1).  QK_j(t+1) reuses
        // S_j's columns, which hold P_j(t): it is issued after PV_j(t).
        if (lane == 0) {
            const uint32_t idesc_qk = kF8 ? idesc_e4m3_f32(128, 128) : idesc_bf16_f32(128, 128, 0, 0);
            const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            int npv[kQT] = {0, 0};
            bool live = !*abort && mbar_wait(&sm.bar_q, 0, abort, p.dev_err);
            // S_j = Q_j K^T for the key tile in ring slot `ks`
            auto issue_qk = [&](int j, uint32_t ka) {
                tc_fence_after();
                const uint32_t qa = smem_u32(sm.q[j]);
                if constexpr (kF8) {
                    // 128 one-byte columns per row: four K = 32 steps within one swizzle atom
#pragma unroll
                    for (int kk = 0; kk < kD / 32; ++kk)
                        umma_ss_f8(tmem + j * 128, smem_desc_sw128(qa + kk * 32, 16, 1024),
                                   smem_desc_sw128(ka + kk * 32, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                } else {
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk < 4) ? kk * 32 : kHalfBytes + (kk - 4) * 32;
                        umma_ss(tmem + j * 128, smem_desc_sw128(qa + off, 16, 1024),
                                smem_desc_sw128(ka + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                    }
                }
                umma_commit(&sm.bar_s[j]);
            };
            if (live && nkt > 0) {
                live = mbar_wait(&sm.full[0], 0, abort, p.dev_err);
                if (live) {
                    const uint32_t ka = smem_u32(sm.kv[0]);
#pragma unroll
                    for (int j = 0; j < kQT; ++j)
                        if (sm.kt[0].use[j]) issue_qk(j, ka);
                    umma_commit(&sm.empty[0]);
                }
            }
            for (int t = 0; t < nkt && live; ++t) {
                const KeyTile kt = sm.kt[t];
                const int uv = 2 * t + 1, sv = uv % kSlots;
                if (!(live = mbar_wait(&sm.full[sv], (uv / kSlots) & 1, abort, p.dev_err))) break;
                const uint32_t va = smem_u32(sm.kv[sv]);
                const bool more = t + 1 < nkt;
                const int uk = 2 * (t + 1), sk = uk % kSlots;
                bool k_ready = false;
#pragma unroll
                for (int j = 0; j < kQT; ++j) {
                    if (kt.use[j]) {
                        if (!(live = mbar_wait(&sm.bar_p[j], npv[j] & 1, abort, p.dev_err))) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk)
                            umma_ts(tmem + 256 + j * 128, tmem + j * 128 + kk * 8,
                                    smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024), idesc_pv,
                                    (npv[j] > 0 || kk > 0) ? 1u : 0u);
                        ++npv[j];
                    }
                    if (more && sm.kt[t + 1].use[j]) {
                        if (!k_ready) {
                            if (!(live = mbar_wait(&sm.full[sk], (uk / kSlots) & 1, abort, p.dev_err))) break;
                            k_ready = true;
                        }
                        issue_qk(j, smem_u32(sm.kv[sk]));
                    }
                }
                if (!live) break;
                umma_commit(&sm.empty[sv]);
                if (more) {
                    // a K tile no query tile uses still has to be released
                    if (!k_ready && !(live = mbar_wait(&sm.full[sk], (uk / kSlots) & 1, abort, p.dev_err))) break;
                    umma_commit(&sm.empty[sk]);
                }
            }
            // every MMA of this CTA is complete once bar_o fires
            umma_commit(&sm.bar_o);
            if (*abort) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                mbar_wait(&sm.bar_o, 0, no_abort, nullptr);
            }
        }
    } else {
        // ------------------------------------------------ softmax + epilogue of tile j
        const int j = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t colS = j * 128, colO = 256 + j * 128;
        const int nqj = j == 0 ? nq0 : nq1;
        const int r_q = r_min + j * kBM + row;
        const float sq = (kF8 && nqj > 0) ? p.sq[((size_t)(b * p.Fseg + seg_f) * p.H + h) * p.nblk + (s0 + j * kBM) / kBM]
                                          : 1.f;
        float m_ref = -INFINITY, l_run = 0.f;
        int n = 0;
        bool ok = !*abort;
        for (int t = 0; t < nkt && ok; ++t) {
            const KeyTile &ktr = sm.kt[t];
            if (!ktr.use[j]) continue;
            const bool full = ktr.full[j];
            const int rbase = ktr.rbase, kvalid = ktr.kvalid;
            // logits scale: log2(e)/sqrt(d), times the e4m3 tiles' scales
            const float sl2 = kF8 ? p.scale_log2 * sq * ktr.sk : p.scale_log2;
            // waits are made warp-uniform: the TMEM loads below are warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_s[j], n & 1, abort, p.dev_err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s[128];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tmem_ld32(tl + colS + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * i]));
            tmem_wait_ld();
            if (!full) {
                const int lo = max(0, r_q - p.w + 1 - rbase);
                const int hi = min(kvalid - 1, r_q + p.w_hi - rbase);
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c < lo || c > hi) s[c] = __float_as_uint(-INFINITY);
            }
            // the softmax scale is positive: take the maximum of the raw scores
            float mx;
            {
                float mm8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mm8[i] = __uint_as_float(s[i]);
#pragma unroll
                for (int c = 8; c < 128; c += 16)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        mm8[i] = max3f(mm8[i], __uint_as_float(s[c + i]), __uint_as_float(s[c + 8 + i]));
                mx = max3f(max3f(mm8[0], mm8[1], mm8[2]), max3f(mm8[3], mm8[4], mm8[5]), fmaxf(mm8[6], mm8[7]));
                mx *= sl2;  // -inf stays -inf
            }
            float alpha = 1.f;
            bool moved = false;
            if (mx > m_ref + kRescaleThreshold) {
                alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mx);
                m_ref = mx;
                moved = true;
            }
            const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
            // P = 2^(s*scale - m) as bf16 over columns 0-63 of S_j
            float sum[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) sum[i] = 0.f;
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float p0 = ex2(fmaf(__uint_as_float(s[hlf * 64 + c]), sl2, neg_m));
                    const float p1 = ex2(fmaf(__uint_as_float(s[hlf * 64 + c + 1]), sl2, neg_m));
                    sum[(c >> 1) & 7] += p0 + p1;
                    pk[c >> 1] = pack_bf16x2(p0, p1);
                }
                tmem_st32(tl + colS + hlf * 32, pk);
            }
            // O_j holds earlier tiles' contributions once n > 0; PV_j(t-1) is complete
            // (it was issued before QK_j(t), whose commit fired)
            if (n > 0 && __any_sync(0xffffffffu, moved)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tl + colO + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) o[jj] = __float_as_uint(__uint_as_float(o[jj]) * alpha);
                    tmem_st32(tl + colO + c * 32, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_p[j]);
            l_run = fmaf(l_run, alpha,
                         ((sum[0] + sum[1]) + (sum[2] + sum[3])) + ((sum[4] + sum[5]) + (sum[6] + sum[7])));
            ++n;
        }
        if (ok && n > 0 && __all_sync(0xffffffffu, mbar_wait(&sm.bar_o, 0, abort, p.dev_err))) {
            tc_fence_after();
            const int tok = seg_f * p.Pseg + s0 + j * kBM + row;
            const size_t base = (((size_t)b * p.L + tok) * p.H + h) * kD;
            const float scale = p.gates[h * 3 + p.gate_col] / l_run;
            if (p.lse_out && row < nqj) p.lse_out[((size_t)b * p.H + h) * p.L + tok] = m_ref + log2f(l_run);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(tl + colO + c * 32, r);
                tmem_wait_ld();
                if (row < nqj) store_chunk(p, base, c * 32, r, scale);
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

// e4m3 quantization of q or k for the FP8 Q K^T path: one CTA per (128-row
// block, head, segment), one thread per row.  scale = max |x| / 448 over the
// 128 x 128 tile (448: the largest finite e4m3 value); x8 = e4m3(x / scale),
// rounded to nearest and saturating.  Rows past the segment end are not
// written (the kernel's tensor map never reads them).
__global__ void __launch_bounds__(128) quant_e4m3_kernel(const __nv_bfloat16 *x, uint8_t *x8, float *scales,
                                                         int Pseg, int H, int nblk) {
    const int blk = blockIdx.x, h = blockIdx.y, seg = blockIdx.z;
    const int r = blk * kBM + threadIdx.x;
    const bool live = r < Pseg;
    const size_t row = ((size_t)seg * Pseg + (live ? r : 0)) * H + h;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + row * kD);
    float v[kD];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < kD / 8; ++c) {
        uint4 u = live ? src[c] : make_uint4(0, 0, 0, 0);
        const __nv_bfloat162 *pr = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[8 * c + 2 * e] = __low2float(pr[e]);
            v[8 * c + 2 * e + 1] = __high2float(pr[e]);
            amax = fmaxf(amax, fmaxf(fabsf(v[8 * c + 2 * e]), fabsf(v[8 * c + 2 * e + 1])));
        }
    }
    __shared__ float wmax[4];
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
    const float scale = amax > 0.f ? amax / 448.f : 1.f;
    const float inv = 1.f / scale;
    if (threadIdx.x == 0) scales[((size_t)seg * H + h) * nblk + blk] = scale;
    if (!live) return;
    uint4 *dst = reinterpret_cast<uint4 *>(x8 + row * kD);
#pragma unroll
    for (int c = 0; c < kD / 16; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = 16 * c + 4 * e;
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[i] * inv, v[i + 1] * inv), __NV_SATFINITE,
                                                         __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v[i + 2] * inv, v[i + 3] * inv),
                                                         __NV_SATFINITE, __NV_E4M3);
            w[e] = lo | (hi << 16);
        }
        dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
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

// 4-D view (d, H, Pseg, B*Fseg) of a [B, L, H, d] bf16 tensor, box (64, 1, 128, 1).
bool make_map(CUtensorMap *map, const void *base, int H, int Pseg, int segs) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)Pseg, (cuuint64_t)segs};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)Pseg * H * kD * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBN, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D view (d, H, Pseg, B*Fseg) of a [B, L, H, d] e4m3 tensor, box (128, 1, 128, 1):
// one 128-byte swizzle atom per row.
bool make_map8(CUtensorMap *map, const void *base, int H, int Pseg, int segs) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)Pseg, (cuuint64_t)segs};
    const cuuint64_t strides[3] = {(cuuint64_t)kD, (cuuint64_t)H * kD, (cuuint64_t)Pseg * H * kD};
    const cuuint32_t box[4] = {(cuuint32_t)kD, 1, (cuuint32_t)kBN, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

class TcAttentionImpl : public TcAttention {
public:
    explicit TcAttentionImpl(const hlta_config &c) : cfg_(c) {}

    // Segment geometry of a branch, or false when this kernel does not take it.
    static bool geometry(int L, WindowGeom g, int *Pseg, int *Fseg) {
        if (g.dil == 1) {
            *Pseg = L;
            *Fseg = 1;
        } else {
            if (L % g.P != 0) return false;  // ragged last frame: CUDA-core kernel
            *Pseg = g.P;
            *Fseg = L / g.P;
        }
        if (*Pseg < kBN) return false;
        // key tiles one CTA can need: the span w + 2*kBM - 1 rearranged rows, cut
        // at most at every segment boundary it crosses
        const long long span = (long long)g.w + g.w_hi + kQT * kBM - 1;
        const long long bound = (span + kBN - 1) / kBN + 2 * (span / *Pseg + 2);
        if (bound > kMaxKT) return false;
        return (long long)*Fseg * *Pseg <= (1LL << 30);
    }

    bool covers(int L, WindowGeom g) const override {
        int a, b;
        return geometry(L, g, &a, &b);
    }

    cudaError_t run(const void *q, const void *k, const void *v, int L, WindowGeom g, const float *gates,
                    int gate_col, int mode, float *acc, const float *acc2, void *out, int *dev_err,
                    cudaStream_t s, bool *done, float *lse_out, const Fp8Scratch *f8) override {
        *done = false;
        int Pseg, Fseg;
        if (!geometry(L, g, &Pseg, &Fseg)) return cudaSuccess;

        CUtensorMap mq, mk, mv;
        const int segs = cfg_.B * Fseg;
        const int nblk = (Pseg + kBM - 1) / kBM;
        if (f8) {
            const dim3 qgrid(nblk, cfg_.H, segs);
            quant_e4m3_kernel<<<qgrid, 128, 0, s>>>(static_cast<const __nv_bfloat16 *>(q),
                                                   static_cast<uint8_t *>(f8->q8), f8->sq, Pseg, cfg_.H, nblk);
            quant_e4m3_kernel<<<qgrid, 128, 0, s>>>(static_cast<const __nv_bfloat16 *>(k),
                                                   static_cast<uint8_t *>(f8->k8), f8->sk, Pseg, cfg_.H, nblk);
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        if (!(f8 ? make_map8(&mq, f8->q8, cfg_.H, Pseg, segs) && make_map8(&mk, f8->k8, cfg_.H, Pseg, segs)
                 : make_map(&mq, q, cfg_.H, Pseg, segs) && make_map(&mk, k, cfg_.H, Pseg, segs)) ||
            !make_map(&mv, v, cfg_.H, Pseg, segs))
            return cudaErrorInvalidValue;
        TcAttnParams p;
        p.Pseg = Pseg;
        p.Fseg = Fseg;
        p.dil = g.dil;
        p.w = g.w;
        p.w_hi = g.w_hi;
        p.qblocks_per_seg = (Pseg + kQT * kBM - 1) / (kQT * kBM);
        p.H = cfg_.H;
        p.L = L;
        p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
        p.gates = gates;
        p.gate_col = gate_col;
        p.out_mode = mode;
        p.acc = acc;
        p.acc2 = acc2;
        p.out = static_cast<__nv_bfloat16 *>(out);
        p.dev_err = dev_err;
        p.lse_out = lse_out;
        p.sq = f8 ? f8->sq : nullptr;
        p.sk = f8 ? f8->sk : nullptr;
        p.nblk = nblk;
        const size_t smem = sizeof(Smem) + 1024;
        if (!attr_set_) {
            cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<false>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
            if (e != cudaSuccess) return e;
            attr_set_ = true;
        }
        const dim3 grid(Fseg * p.qblocks_per_seg, cfg_.H, cfg_.B);
        if (f8)
            attn_tc_kernel<true><<<grid, kThreads, smem, s>>>(mq, mk, mv, p);
        else
            attn_tc_kernel<false><<<grid, kThreads, smem, s>>>(mq, mk, mv, p);
        *done = true;
        return cudaGetLastError();
    }

private:
    hlta_config cfg_;
    bool attr_set_ = false;
};

}  // namespace

size_t fp8_scale_floats(int B, int H, int max_len, int tokens_per_frame) {
    const size_t swa = (size_t)(max_len + kBM - 1) / kBM;
    const size_t frames = (size_t)max_len / tokens_per_frame + 1;
    const size_t dswa = frames * (size_t)((tokens_per_frame + kBM - 1) / kBM);
    return (size_t)B * H * (swa > dswa ? swa : dswa);
}

TcAttention *TcAttention::create(const hlta_config &cfg, long long) {
    if (cfg.dtype != HLTA_BF16 || cfg.d_k != kD || cfg.d_v != kD) return nullptr;
    return new TcAttentionImpl(cfg);
}

}  // namespace hlta
