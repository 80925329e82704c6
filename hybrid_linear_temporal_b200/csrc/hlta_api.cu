// hlta_api.cu -- the C ABI declared in include/hlta.h: argument checks,
// handle-owned device memory, and the launch sequence of one layer pass.
//
// One pass (Kairos paper, section 2.2) runs the selected branches in the order
// GDN, SWA, DSWA on the caller's stream.  Each branch kernel adds its gated
// output g[h,b]*o_b into an fp32 accumulator; the last one selected writes the
// layer output in the configured dtype (fused gate/sum epilogue).
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <string>
#include <vector>

#include "hlta.h"
#include "kernels.h"
#include "tc_attention.h"
#include "tc_attn_bwd.h"
#include "tc_gdn.h"

namespace {

thread_local std::string g_last_error;

hlta_status fail(hlta_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

hlta_status ok() {
    g_last_error.clear();
    return HLTA_OK;
}

// Host-side failure injection for tests: HLTA_INJECT_FAIL=<entry point name>
// (or "all") makes that entry point fail with HLTA_ERR_INJECTED before doing
// anything.
bool injected(const char *fn) {
    const char *e = getenv("HLTA_INJECT_FAIL");
    if (!e || !*e) return false;
    return strcmp(e, "all") == 0 || strcmp(e, fn) == 0;
}

#define INJECT(fn)                                                        \
    do {                                                                  \
        if (injected(fn)) return fail(HLTA_ERR_INJECTED, "%s: injected failure", fn); \
    } while (0)

#define CK(call)                                                                          \
    do {                                                                                  \
        cudaError_t e_ = (call);                                                          \
        if (e_ != cudaSuccess)                                                            \
            return fail(HLTA_ERR_CUDA, "%s:%d %s: %s", __FILE__, __LINE__, #call,        \
                        cudaGetErrorString(e_));                                          \
    } while (0)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace hlta {
// Sets the thread-local message returned by hlta_last_error() (empty clears it).
void set_last_error(const char *msg) { g_last_error = msg ? msg : ""; }
}  // namespace hlta

struct hlta_handle {
    hlta_config cfg;
    int device = 0;
    int elem_bytes = 2;
    long long acc_rows = 0;      // token rows per batch the accumulator holds
    float *acc = nullptr;        // [B, acc_rows, H, d_v]
    int *dev_err = nullptr;      // device error word
    // streaming state
    float *S_stream = nullptr;   // [B, H, d_v, d_k]
    void *ring_k = nullptr;      // [B, ring_cap, H, d_k]
    void *ring_v = nullptr;      // [B, ring_cap, H, d_v]
    long long ring_cap = 0;
    long long pos = 0;
    long long hdr[8] = {0};
    // staging for hlta_forward_host
    char *stage = nullptr;
    size_t stage_bytes = 0;
    hlta::TcAttention *tc_attn = nullptr;
    hlta::TcGdn *tc_gdn = nullptr;
    // concurrent memory branch: side stream, fork/join events, its own accumulator
    cudaStream_t side = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    float *acc2 = nullptr;
    // rotated q and k for the attention branches (rope_base > 0)
    void *q_rot = nullptr, *k_rot = nullptr;
    // e4m3 copies of q and k and their tile scales (attn_fp8)
    hlta::Fp8Scratch f8 = {nullptr, nullptr, nullptr, nullptr};
    // backward scratch: one block allocated at the first hlta_backward, kept
    char *bw_block = nullptr;
    float *g_dq = nullptr, *g_dk = nullptr, *g_dv = nullptr, *g_dq_att = nullptr, *g_dk_att = nullptr;
    float *g_lse = nullptr, *g_rowdot[3] = {nullptr, nullptr, nullptr}, *g_rowdot_hm = nullptr;
    float *g_ones = nullptr;  // [H, 3] gates of one: the forward writes the ungated branch output
    hlta::TcAttnBwd *tc_bwd = nullptr;
    float *bw_W = nullptr, *bw_TbV = nullptr, *bw_Kd = nullptr, *bw_T = nullptr, *bw_Lc = nullptr;
    float *bw_ell = nullptr, *bw_S = nullptr, *bw_dS = nullptr, *bw_U = nullptr, *bw_ws = nullptr;
    size_t bw_ws_floats = 0;
    int bw_grid = 0;
    // profiling (hlta_profile_enable)
    bool prof = false;
    struct Mark {
        int slot;
        cudaEvent_t a, b;
    };
    std::vector<Mark> marks;
    std::vector<cudaEvent_t> event_pool;
    double prof_ms[3] = {0, 0, 0};
    long long prof_passes[3] = {0, 0, 0};
    long long prof_launches = 0;
};

namespace {

constexpr long long kCkptMagic = 0x484c544143503031LL;  // "HLTACP01"
constexpr size_t kCkptHeader = 256;

size_t state_elems(const hlta_config &c) { return (size_t)c.B * c.H * c.d_v * c.d_k; }

// Farthest key (in tokens, behind the query) any window can admit.
long long max_lookback(const hlta_config &c) {
    const long long P = c.tokens_per_frame;
    const long long swa = c.swa_window - 1;
    // DSWA: i - j = dil*g*P + s_i - s_j with r(i) - r(j) = g*P + s_i - s_j < w and
    // g*P <= w - 1 + P - 1, so i - j <= (dil - 1)*g_max*P + w - 1.
    const long long gmax = (c.dswa_window + P - 2) / P;
    const long long dswa = (long long)(c.dswa_dilation - 1) * gmax * P + c.dswa_window - 1;
    return swa > dswa ? swa : dswa;
}

hlta_status check_config(const hlta_config *c) {
    if (!c) return fail(HLTA_ERR_INVALID_ARG, "hlta_create: cfg is NULL");
    if (c->B < 1 || c->H < 1) return fail(HLTA_ERR_INVALID_ARG, "B and H must be >= 1");
    if (c->d_k < 1 || c->d_v < 1) return fail(HLTA_ERR_INVALID_ARG, "d_k and d_v must be >= 1");
    if (c->tokens_per_frame < 1) return fail(HLTA_ERR_INVALID_ARG, "tokens_per_frame must be >= 1");
    if (c->swa_window < 1 || c->dswa_window < 1)
        return fail(HLTA_ERR_INVALID_ARG, "windows must be >= 1");
    if (c->dswa_dilation < 1) return fail(HLTA_ERR_INVALID_ARG, "dswa_dilation must be >= 1");
    if (c->dtype != HLTA_BF16 && c->dtype != HLTA_FP32)
        return fail(HLTA_ERR_INVALID_ARG, "dtype must be HLTA_BF16 or HLTA_FP32");
    if (c->max_seq_len < 1) return fail(HLTA_ERR_INVALID_ARG, "max_seq_len must be >= 1");
    if (c->max_stream_tokens < 0) return fail(HLTA_ERR_INVALID_ARG, "max_stream_tokens must be >= 0");
    if (c->gdn_form != HLTA_GDN_DECAYED && c->gdn_form != HLTA_GDN_PAGES)
        return fail(HLTA_ERR_INVALID_ARG, "gdn_form must be HLTA_GDN_DECAYED or HLTA_GDN_PAGES");
    if (c->window_mode != HLTA_WINDOW_CAUSAL && c->window_mode != HLTA_WINDOW_CENTRED)
        return fail(HLTA_ERR_INVALID_ARG, "window_mode must be HLTA_WINDOW_CAUSAL or HLTA_WINDOW_CENTRED");
    if (!(c->rope_base >= 0.f) || c->rope_base > 1e30f)
        return fail(HLTA_ERR_INVALID_ARG, "rope_base must be a finite value >= 0");
    if (c->window_mode == HLTA_WINDOW_CENTRED && c->max_stream_tokens > 0)
        return fail(HLTA_ERR_UNSUPPORTED, "centred windows need the whole sequence: not with streaming");
    if (c->rope_base > 0.f && c->window_mode != HLTA_WINDOW_CENTRED)
        return fail(HLTA_ERR_UNSUPPORTED, "rotary embedding is provided with centred windows");
    if (c->attn_fp8 != 0 && c->attn_fp8 != 1) return fail(HLTA_ERR_INVALID_ARG, "attn_fp8 must be 0 or 1");
    if (c->attn_fp8 && (c->dtype != HLTA_BF16 || c->d_k != 128 || c->d_v != 128))
        return fail(HLTA_ERR_UNSUPPORTED, "attn_fp8 needs dtype HLTA_BF16 and d_k = d_v = 128");
    if ((c->d_k != 64 && c->d_k != 128) || (c->d_v != 64 && c->d_v != 128))
        return fail(HLTA_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128");
    if (c->chunk != 64) return fail(HLTA_ERR_UNSUPPORTED, "chunk must be 64");
    const long long big = 1LL << 31;
    if ((long long)c->B * c->max_seq_len * c->H >= big / 128)
        return fail(HLTA_ERR_UNSUPPORTED, "B*max_seq_len*H too large");
    return HLTA_OK;
}

struct Inputs {
    const void *q, *k, *v;
    const float *alpha, *beta, *gates;
};

hlta_status check_inputs(const char *fn, const Inputs &in, const void *out) {
    const void *ptrs[] = {in.q, in.k, in.v, in.alpha, in.beta, in.gates, out};
    const char *names[] = {"q", "k", "v", "alpha", "beta", "gates", "out"};
    for (int i = 0; i < 7; ++i) {
        if (!ptrs[i]) return fail(HLTA_ERR_INVALID_ARG, "%s: %s is NULL", fn, names[i]);
        if (!aligned16(ptrs[i]))
            return fail(HLTA_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, names[i]);
    }
    return HLTA_OK;
}

cudaEvent_t pooled_event(hlta_handle *h) {
    if (!h->event_pool.empty()) {
        cudaEvent_t e = h->event_pool.back();
        h->event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Brackets one branch's launches with events when profiling is on.
struct ProfScope {
    hlta_handle *h;
    int slot;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    ProfScope(hlta_handle *h_, int slot_, cudaStream_t s_) : h(h_), slot(slot_), s(s_) {
        if (!h->prof) return;
        a = pooled_event(h);
        b = pooled_event(h);
        if (a && b) cudaEventRecord(a, s);
    }
    void done(int launches) {
        if (!h->prof || !a || !b) return;
        cudaEventRecord(b, s);
        h->marks.push_back({slot, a, b});
        h->prof_launches += launches;
    }
};

// Output mode of the idx-th of n selected branches.
int out_mode(int idx, int n) {
    if (n == 1) return hlta::OUT_FINAL_ONLY;
    if (idx == 0) return hlta::OUT_STORE;
    return idx == n - 1 ? hlta::OUT_FINAL : hlta::OUT_ADD;
}

// Window geometry of attention branch br (0 = SWA, 1 = DSWA).
hlta::WindowGeom window_of(const hlta_config &c, int br) {
    hlta::WindowGeom g;
    g.P = c.tokens_per_frame;
    g.dil = br == 0 ? 1 : c.dswa_dilation;
    const int w = br == 0 ? c.swa_window : c.dswa_window;
    if (c.window_mode == HLTA_WINDOW_CENTRED) {
        g.w = w / 2 + 1;  // r - w/2 <= r_k
        g.w_hi = w / 2;   // r_k <= r + w/2
    } else {
        g.w = w;
        g.w_hi = 0;
    }
    return g;
}

// Run the selected branches of one pass.
//   nq queries at absolute positions pos0 .. pos0+nq-1 (q, alpha, beta, k, v of
//   those tokens: [B, nq, ...]); keys/values are read from (kst, vst) with
//   key_rows rows per batch (position p at row p % key_rows).
hlta_status run_pass(hlta_handle *h, const Inputs &in, long long pos0, int nq, const void *kst,
                     const void *vst, long long key_rows, bool one_shot, const float *S_in,
                     float *S_out, void *out, unsigned branches, cudaStream_t s) {
    const hlta_config &c = h->cfg;
    const bool bf16 = c.dtype == HLTA_BF16;
    // Order: memory first (its per-token column writes only store), then SWA,
    // then DSWA, whose epilogue reads the accumulator row by row and writes out.
    const int order[3] = {2, 0, 1};
    int sel[3], n = 0;
    for (int i = 0; i < 3; ++i)
        if (branches & (1u << order[i])) sel[n++] = order[i];
    if (n == 0) {
        CK(cudaMemsetAsync(out, 0, (size_t)c.B * nq * c.H * c.d_v * h->elem_bytes, s));
        return HLTA_OK;
    }
    const hlta::WindowGeom geo[2] = {window_of(c, 0), window_of(c, 1)};
    const bool want_attn[2] = {(branches & 1u) != 0, (branches & 2u) != 0};
    // the attention branches read rotated q and k when rotary embedding is on
    // (one-shot passes only: centred windows exclude streaming)
    Inputs att = in;
    if (c.rope_base > 0.f && (want_attn[0] || want_attn[1])) {
        hlta::RopeArgs r;
        r.q = in.q;
        r.k = kst;
        r.q_out = h->q_rot;
        r.k_out = h->k_rot;
        r.B = c.B;
        r.n = nq;
        r.H = c.H;
        r.d = c.d_k;
        r.pos0 = pos0;
        for (int m = 0; m < 64; ++m) r.inv_freq[m] = m < c.d_k / 2 ? pow((double)c.rope_base, -2.0 * m / c.d_k) : 0.0;
        CK(hlta::launch_rope(r, bf16, s));
        if (h->prof) h->prof_launches += 1;
        att.q = h->q_rot;
        kst = h->k_rot;
    }
    // Concurrent schedule: the memory branch (prep kernels and a sequential
    // scan on B*H SMs) runs on the side stream into its own accumulator while
    // the first attention branch runs on `s`; the last attention branch waits
    // for the memory branch and its epilogue writes out = acc + acc2 + its own
    // gated output (the gated sum of all three branches).
    const bool overlap = one_shot && (branches & 4u) && (want_attn[0] || want_attn[1]) && h->side &&
                         h->acc2 && h->tc_gdn && h->tc_gdn->covers(nq) && h->tc_attn &&
                         (!want_attn[0] || h->tc_attn->covers(nq, geo[0])) &&
                         (!want_attn[1] || h->tc_attn->covers(nq, geo[1]));
    if (overlap) {
        CK(cudaEventRecord(h->ev_fork, s));
        CK(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
        {
            ProfScope ps(h, 2, h->side);
            bool done = false;
            int launches = 1;
            cudaError_t e = h->tc_gdn->run(in.q, in.k, in.v, in.alpha, in.beta, nq, S_in, S_out, in.gates,
                                           hlta::OUT_STORE, h->acc2, out, h->dev_err, h->side, &done,
                                           &launches);
            if (e != cudaSuccess || !done)
                return fail(HLTA_ERR_CUDA, "tensor-core memory: %s", cudaGetErrorString(e));
            ps.done(launches);
        }
        CK(cudaEventRecord(h->ev_join, h->side));
        // attention on `s` beside the memory branch; the last attention branch
        // joins it and finishes the output
        const int n_attn = (want_attn[0] ? 1 : 0) + (want_attn[1] ? 1 : 0);
        int idx = 0;
        for (int br = 0; br < 2; ++br) {
            if (!want_attn[br]) continue;
            const bool last = idx == n_attn - 1;
            if (last) CK(cudaStreamWaitEvent(s, h->ev_join, 0));
            ProfScope ps(h, br, s);
            bool done = false;
            const int mode = last ? (idx == 0 ? hlta::OUT_FINAL_ONLY : hlta::OUT_FINAL) : hlta::OUT_STORE;
            cudaError_t e = h->tc_attn->run(att.q, kst, vst, nq, geo[br], in.gates, br, mode, h->acc,
                                            last ? h->acc2 : nullptr, out, h->dev_err, s, &done, nullptr,
                                            c.attn_fp8 ? &h->f8 : nullptr);
            if (e != cudaSuccess || !done)
                return fail(HLTA_ERR_CUDA, "tensor-core attention: %s", cudaGetErrorString(e));
            ps.done(1);
            ++idx;
        }
        return HLTA_OK;
    }
    for (int idx = 0; idx < n; ++idx) {
        const int br = sel[idx];
        const int mode = out_mode(idx, n);
        ProfScope ps(h, br, s);
        int launches = 1;
        if (br == 0 || br == 1) {
            const hlta::WindowGeom g = geo[br];
            bool done = false;
            if (one_shot && h->tc_attn) {
                cudaError_t e = h->tc_attn->run(att.q, kst, vst, nq, g, in.gates, br, mode, h->acc,
                                                nullptr, out, h->dev_err, s, &done, nullptr,
                                                c.attn_fp8 ? &h->f8 : nullptr);
                if (e != cudaSuccess)
                    return fail(HLTA_ERR_CUDA, "tensor-core attention: %s", cudaGetErrorString(e));
            }
            if (!done) {
                hlta::AttnSimtArgs a;
                a.q = att.q;
                a.k = kst;
                a.v = vst;
                a.q_pos0 = pos0;
                a.nq = nq;
                a.B = c.B;
                a.H = c.H;
                a.d_k = c.d_k;
                a.d_v = c.d_v;
                a.key_rows = key_rows;
                a.n_keys = pos0 + nq;
                a.geom = g;
                a.scale_log2 = 1.4426950408889634f / sqrtf((float)c.d_k);
                a.gates = in.gates;
                a.gate_col = br;
                a.out_mode = mode;
                a.acc = h->acc;
                a.out = out;
                CK(hlta::launch_attn_simt(a, bf16, s));
            }
        } else {
            bool done = false;
            if (h->tc_gdn) {
                cudaError_t e = h->tc_gdn->run(in.q, in.k, in.v, in.alpha, in.beta, nq, S_in, S_out,
                                               in.gates, mode, h->acc, out, h->dev_err, s, &done,
                                               &launches);
                if (e != cudaSuccess)
                    return fail(HLTA_ERR_CUDA, "tensor-core memory: %s", cudaGetErrorString(e));
            }
            if (!done) {
                hlta::GdnRecArgs a;
                a.q = in.q;
                a.k = in.k;
                a.v = in.v;
                a.alpha = in.alpha;
                a.beta = in.beta;
                a.S_in = S_in;
                a.S_out = S_out;
                a.n = nq;
                a.B = c.B;
                a.H = c.H;
                a.d_k = c.d_k;
                a.d_v = c.d_v;
                a.gates = in.gates;
                a.out_mode = mode;
                a.acc = h->acc;
                a.out = out;
                a.form = c.gdn_form;
                CK(hlta::launch_gdn_recurrent(a, bf16, s));
            }
        }
        ps.done(launches);
    }
    return HLTA_OK;
}

}  // namespace

extern "C" {

int hlta_version(void) { return 100; }

const char *hlta_last_error(void) { return g_last_error.c_str(); }

hlta_status hlta_create(const hlta_config *cfg, hlta_handle **out) {
    INJECT("hlta_create");
    if (!out) return fail(HLTA_ERR_INVALID_ARG, "hlta_create: out is NULL");
    *out = nullptr;
    hlta_status st = check_config(cfg);
    if (st != HLTA_OK) return st;

    int dev = 0;
    CK(cudaGetDevice(&dev));
    cudaDeviceProp prop;
    CK(cudaGetDeviceProperties(&prop, dev));
    if (prop.major != 10)
        return fail(HLTA_ERR_CUDA, "hlta_create: device %d is sm_%d%d; this build targets sm_100a",
                    dev, prop.major, prop.minor);

    hlta_handle *h = new hlta_handle();
    h->cfg = *cfg;
    h->device = dev;
    h->elem_bytes = cfg->dtype == HLTA_BF16 ? 2 : 4;
    h->acc_rows = cfg->max_seq_len > cfg->max_stream_tokens ? cfg->max_seq_len : cfg->max_stream_tokens;

    auto alloc = [&](void **p, size_t bytes) -> bool {
        if (cudaMalloc(p, bytes) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        return true;
    };
    const size_t acc_bytes = (size_t)cfg->B * h->acc_rows * cfg->H * cfg->d_v * sizeof(float);
    bool okk = alloc((void **)&h->acc, acc_bytes) && alloc((void **)&h->dev_err, sizeof(int));
    if (okk && cfg->attn_fp8) {
        const size_t n8 = (size_t)cfg->B * cfg->max_seq_len * cfg->H * 128;
        const size_t ns = hlta::fp8_scale_floats(cfg->B, cfg->H, cfg->max_seq_len, cfg->tokens_per_frame);
        okk = alloc(&h->f8.q8, n8) && alloc(&h->f8.k8, n8) && alloc((void **)&h->f8.sq, ns * sizeof(float)) &&
              alloc((void **)&h->f8.sk, ns * sizeof(float));
    }
    if (okk && cfg->rope_base > 0.f) {
        const size_t qk_bytes = (size_t)cfg->B * cfg->max_seq_len * cfg->H * cfg->d_k * h->elem_bytes;
        okk = alloc(&h->q_rot, qk_bytes) && alloc(&h->k_rot, qk_bytes);
    }
    if (okk && cfg->max_stream_tokens > 0) {
        long long cap = cfg->max_stream_tokens + max_lookback(*cfg);
        cap = (cap + 127) / 128 * 128;
        h->ring_cap = cap;
        okk = alloc((void **)&h->S_stream, state_elems(*cfg) * sizeof(float)) &&
              alloc(&h->ring_k, (size_t)cfg->B * cap * cfg->H * cfg->d_k * h->elem_bytes) &&
              alloc(&h->ring_v, (size_t)cfg->B * cap * cfg->H * cfg->d_v * h->elem_bytes);
    }
    if (!okk) {
        hlta_destroy(h);
        return fail(HLTA_ERR_OOM, "hlta_create: device allocation failed");
    }
    if (cudaMemset(h->dev_err, 0, sizeof(int)) != cudaSuccess ||
        (h->S_stream && cudaMemset(h->S_stream, 0, state_elems(*cfg) * sizeof(float)) != cudaSuccess)) {
        hlta_destroy(h);
        return fail(HLTA_ERR_CUDA, "hlta_create: cudaMemset failed");
    }
    if (cfg->dtype == HLTA_BF16) {
        h->tc_attn = hlta::TcAttention::create(*cfg, h->acc_rows);
        h->tc_gdn = hlta::TcGdn::create(*cfg, cfg->max_seq_len);
        if (h->tc_attn && h->tc_gdn) {
            const size_t acc2_bytes = (size_t)cfg->B * cfg->max_seq_len * cfg->H * cfg->d_v * sizeof(float);
            // the memory branch is latency-bound and on the critical path: its stream
            // gets the highest priority so its CTAs are scheduled first as SMs free up
            int prio_lo = 0, prio_hi = 0;
            cudaDeviceGetStreamPriorityRange(&prio_lo, &prio_hi);
            if (cudaStreamCreateWithPriority(&h->side, cudaStreamNonBlocking, prio_hi) != cudaSuccess ||
                cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess ||
                cudaMalloc((void **)&h->acc2, acc2_bytes) != cudaSuccess) {
                cudaGetLastError();
                hlta_destroy(h);
                return fail(HLTA_ERR_OOM, "hlta_create: side stream / accumulator allocation failed");
            }
        }
    }
    *out = h;
    return ok();
}

hlta_status hlta_destroy(hlta_handle *h) {
    if (!h) return ok();
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    cudaFree(h->acc);
    cudaFree(h->dev_err);
    cudaFree(h->S_stream);
    cudaFree(h->ring_k);
    cudaFree(h->ring_v);
    cudaFree(h->stage);
    cudaFree(h->acc2);
    cudaFree(h->q_rot);
    cudaFree(h->k_rot);
    cudaFree(h->bw_block);
    cudaFree(h->f8.q8);
    cudaFree(h->f8.k8);
    cudaFree(h->f8.sq);
    cudaFree(h->f8.sk);
    if (h->side) cudaStreamDestroy(h->side);
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    for (auto &m : h->marks) {
        cudaEventDestroy(m.a);
        cudaEventDestroy(m.b);
    }
    for (auto e : h->event_pool) cudaEventDestroy(e);
    delete h->tc_attn;
    delete h->tc_gdn;
    delete h->tc_bwd;
    delete h;
    return ok();
}

hlta_status hlta_forward(hlta_handle *h, int L, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, const float *gates, const float *S0,
                         float *S_out, void *out, unsigned branches, void *stream) {
    INJECT("hlta_forward");
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_forward: handle is NULL");
    if (L < 1 || L > h->cfg.max_seq_len)
        return fail(HLTA_ERR_INVALID_ARG, "hlta_forward: L=%d outside [1, max_seq_len=%d]", L,
                    h->cfg.max_seq_len);
    if (branches & ~7u) return fail(HLTA_ERR_INVALID_ARG, "hlta_forward: unknown branch bits");
    if (branches == 0) branches = HLTA_BRANCH_ALL;
    Inputs in{q, k, v, alpha, beta, gates};
    hlta_status st = check_inputs("hlta_forward", in, out);
    if (st != HLTA_OK) return st;
    if ((S0 && !aligned16(S0)) || (S_out && !aligned16(S_out)))
        return fail(HLTA_ERR_INVALID_ARG, "hlta_forward: S0/S_out not 16-byte aligned");
    CK(cudaSetDevice(h->device));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = run_pass(h, in, 0, L, k, v, L, true, S0, (branches & HLTA_BRANCH_GDN) ? S_out : nullptr,
                  out, branches, s);
    if (st != HLTA_OK) return st;
    CK(cudaGetLastError());
    return ok();
}

namespace {

// Carves the backward scratch out of one allocation (sizes for max_seq_len).
hlta_status ensure_bwd_scratch(hlta_handle *h) {
    if (h->bw_block) return HLTA_OK;
    const hlta_config &c = h->cfg;
    const size_t rows = (size_t)c.B * c.max_seq_len * c.H, bh = (size_t)c.B * c.H;
    const size_t nc = (size_t)(c.max_seq_len + 63) / 64, ch = bh * nc;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device);
    h->bw_grid = (int)(ch < (size_t)2 * sms ? ch : (size_t)2 * sms);
    h->bw_ws_floats = hlta::gdn_bwd_ws_floats(c.d_k, c.d_v);
    const bool rope = c.rope_base > 0.f;
    std::vector<std::pair<float **, size_t>> parts = {
        {&h->g_dq, rows * c.d_k}, {&h->g_dk, rows * c.d_k}, {&h->g_dv, rows * c.d_v},
        {&h->g_dq_att, rope ? rows * c.d_k : 0}, {&h->g_dk_att, rope ? rows * c.d_k : 0},
        {&h->g_lse, rows}, {&h->g_rowdot[0], rows}, {&h->g_rowdot[1], rows}, {&h->g_rowdot[2], rows},
        {&h->g_rowdot_hm, rows}, {&h->g_ones, (size_t)c.H * 3},
        {&h->bw_W, ch * 64 * c.d_k}, {&h->bw_TbV, ch * 64 * c.d_v}, {&h->bw_Kd, ch * 64 * c.d_k},
        {&h->bw_T, ch * 64 * 64}, {&h->bw_Lc, ch * c.d_v * c.d_k}, {&h->bw_ell, ch * 64},
        {&h->bw_S, ch * c.d_v * c.d_k}, {&h->bw_dS, ch * c.d_v * c.d_k}, {&h->bw_U, ch * 64 * c.d_v},
        {&h->bw_ws, (size_t)h->bw_grid * h->bw_ws_floats}};
    size_t total = 0;
    for (auto &p : parts) total += (p.second * sizeof(float) + 255) / 256 * 256;
    if (cudaMalloc((void **)&h->bw_block, total) != cudaSuccess) {
        cudaGetLastError();
        h->bw_block = nullptr;
        return fail(HLTA_ERR_OOM, "hlta_backward: scratch allocation of %zu bytes failed", total);
    }
    size_t off = 0;
    for (auto &p : parts) {
        *p.first = p.second ? reinterpret_cast<float *>(h->bw_block + off) : nullptr;
        off += (p.second * sizeof(float) + 255) / 256 * 256;
    }
    std::vector<float> ones((size_t)c.H * 3, 1.f);
    CK(cudaMemcpy(h->g_ones, ones.data(), ones.size() * sizeof(float), cudaMemcpyHostToDevice));
    h->tc_bwd = hlta::TcAttnBwd::create(c);
    return HLTA_OK;
}

}  // namespace

hlta_status hlta_backward(hlta_handle *h, int L, const void *q, const void *k, const void *v,
                          const float *alpha, const float *beta, const float *gates, const float *S0,
                          const void *dout, const float *dS_final, void *dq, void *dk, void *dv,
                          float *dalpha, float *dbeta, float *dgates, float *dS0, unsigned branches,
                          void *stream) {
    INJECT("hlta_backward");
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_backward: handle is NULL");
    const hlta_config &c = h->cfg;
    if (L < 1 || L > c.max_seq_len)
        return fail(HLTA_ERR_INVALID_ARG, "hlta_backward: L=%d outside [1, max_seq_len=%d]", L, c.max_seq_len);
    if (branches & ~7u) return fail(HLTA_ERR_INVALID_ARG, "hlta_backward: unknown branch bits");
    if (branches == 0) branches = HLTA_BRANCH_ALL;
    Inputs in{q, k, v, alpha, beta, gates};
    hlta_status st = check_inputs("hlta_backward", in, dout);
    if (st != HLTA_OK) return st;
    const void *outs[] = {dq, dk, dv, dalpha, dbeta, dgates};
    const char *names[] = {"dq", "dk", "dv", "dalpha", "dbeta", "dgates"};
    for (int i = 0; i < 6; ++i) {
        if (!outs[i]) return fail(HLTA_ERR_INVALID_ARG, "hlta_backward: %s is NULL", names[i]);
        if (!aligned16(outs[i]))
            return fail(HLTA_ERR_INVALID_ARG, "hlta_backward: %s is not 16-byte aligned", names[i]);
    }
    if ((S0 && !aligned16(S0)) || (dS_final && !aligned16(dS_final)) || (dS0 && !aligned16(dS0)))
        return fail(HLTA_ERR_INVALID_ARG, "hlta_backward: S0/dS_final/dS0 not 16-byte aligned");
    if ((branches & HLTA_BRANCH_GDN) && c.gdn_form != HLTA_GDN_DECAYED)
        return fail(HLTA_ERR_UNSUPPORTED, "hlta_backward: the memory backward covers gdn_form = HLTA_GDN_DECAYED");
    CK(cudaSetDevice(h->device));
    st = ensure_bwd_scratch(h);
    if (st != HLTA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf16 = c.dtype == HLTA_BF16;
    const size_t rows = (size_t)c.B * L * c.H;

    // memory branch: stores the fp32 gradient accumulators, dalpha, dbeta
    if (branches & HLTA_BRANCH_GDN) {
        hlta::GdnBwdArgs a;
        a.q = q;
        a.k = k;
        a.v = v;
        a.dout = dout;
        a.alpha = alpha;
        a.beta = beta;
        a.gates = gates;
        a.S0 = S0;
        a.dS_final = dS_final;
        a.L = L;
        a.B = c.B;
        a.H = c.H;
        a.d_k = c.d_k;
        a.d_v = c.d_v;
        a.bw_W = h->bw_W;
        a.bw_TbV = h->bw_TbV;
        a.bw_Kd = h->bw_Kd;
        a.bw_T = h->bw_T;
        a.bw_Lc = h->bw_Lc;
        a.bw_ell = h->bw_ell;
        a.bw_S = h->bw_S;
        a.bw_dS = h->bw_dS;
        a.bw_U = h->bw_U;
        a.ws = h->bw_ws;
        a.ws_per_cta = h->bw_ws_floats;
        const long long ch = (long long)c.B * c.H * ((L + 63) / 64);
        a.grid_chunks = (int)(ch < h->bw_grid ? ch : h->bw_grid);
        a.dq = h->g_dq;
        a.dk = h->g_dk;
        a.dv = h->g_dv;
        a.dalpha = dalpha;
        a.dbeta = dbeta;
        a.dS0 = dS0;
        a.rowdot = h->g_rowdot[2];
        CK(hlta::launch_gdn_bwd(a, bf16, s));
    } else {
        CK(cudaMemsetAsync(h->g_dq, 0, rows * c.d_k * sizeof(float), s));
        CK(cudaMemsetAsync(h->g_dk, 0, rows * c.d_k * sizeof(float), s));
        CK(cudaMemsetAsync(h->g_dv, 0, rows * c.d_v * sizeof(float), s));
        CK(cudaMemsetAsync(dalpha, 0, rows * sizeof(float), s));
        CK(cudaMemsetAsync(dbeta, 0, rows * sizeof(float), s));
        if (dS0) CK(cudaMemsetAsync(dS0, 0, state_elems(c) * sizeof(float), s));
    }

    // attention branches: add into the accumulators (rotated-frame dq, dk apart)
    const bool rope = c.rope_base > 0.f && (branches & 3u);
    hlta::BwdFinalizeArgs fq;
    fq.rope = rope ? 1 : 0;
    for (int m = 0; m < 64; ++m)
        fq.inv_freq[m] = rope && m < c.d_k / 2 ? pow((double)c.rope_base, -2.0 * m / c.d_k) : 0.0;
    const void *qa = q, *ka = k;
    float *adq = h->g_dq, *adk = h->g_dk;
    if (rope) {
        hlta::RopeArgs r;
        r.q = q;
        r.k = k;
        r.q_out = h->q_rot;
        r.k_out = h->k_rot;
        r.B = c.B;
        r.n = L;
        r.H = c.H;
        r.d = c.d_k;
        r.pos0 = 0;
        for (int m = 0; m < 64; ++m) r.inv_freq[m] = fq.inv_freq[m];
        CK(hlta::launch_rope(r, bf16, s));
        qa = h->q_rot;
        ka = h->k_rot;
        adq = h->g_dq_att;
        adk = h->g_dk_att;
        CK(cudaMemsetAsync(adq, 0, rows * c.d_k * sizeof(float), s));
        CK(cudaMemsetAsync(adk, 0, rows * c.d_k * sizeof(float), s));
    }
    for (int br = 0; br < 2; ++br) {
        if (!(branches & (1u << br))) continue;
        const hlta::WindowGeom geo = window_of(c, br);
        if (h->tc_attn && h->tc_bwd && h->tc_bwd->covers(L, geo)) {
            // tensor cores: the forward (ungated output and log-sum-exp), dout . o, then dQ and dK/dV
            bool done = false;
            cudaError_t e = h->tc_attn->run(qa, ka, v, L, geo, h->g_ones, br, hlta::OUT_STORE, h->acc, nullptr,
                                            nullptr, h->dev_err, s, &done, h->g_lse);
            if (e != cudaSuccess) return fail(HLTA_ERR_CUDA, "hlta_backward: forward: %s", cudaGetErrorString(e));
            if (done) {
                CK(hlta::launch_rowdot(dout, h->acc, (long long)rows, c.d_v, L, c.H, bf16, h->g_rowdot[br],
                                       h->g_rowdot_hm, s));
                e = h->tc_bwd->run(qa, ka, v, dout, L, geo, gates, br, h->g_lse, h->g_rowdot_hm, adq, adk, h->g_dv,
                                   h->dev_err, s);
                if (e != cudaSuccess)
                    return fail(HLTA_ERR_CUDA, "hlta_backward: tensor-core attention: %s", cudaGetErrorString(e));
                continue;
            }
        }
        hlta::AttnBwdArgs a;
        a.q = qa;
        a.k = ka;
        a.v = v;
        a.dout = dout;
        a.L = L;
        a.B = c.B;
        a.H = c.H;
        a.d_k = c.d_k;
        a.d_v = c.d_v;
        a.geom = geo;
        a.scale_log2 = 1.4426950408889634f / sqrtf((float)c.d_k);
        a.scale = 1.f / sqrtf((float)c.d_k);
        a.gates = gates;
        a.gate_col = br;
        a.lse = h->g_lse;
        a.rowdot = h->g_rowdot[br];
        a.dq = adq;
        a.dk = adk;
        a.dv = h->g_dv;
        CK(hlta::launch_attn_bwd(a, bf16, s));
    }

    // accumulators to the tensor type
    fq.acc = h->g_dq;
    fq.att = rope ? h->g_dq_att : nullptr;
    fq.out = dq;
    fq.rows = (long long)rows;
    fq.d = c.d_k;
    fq.L = L;
    fq.H = c.H;
    CK(hlta::launch_bwd_finalize(fq, bf16, s));
    hlta::BwdFinalizeArgs fk = fq;
    fk.acc = h->g_dk;
    fk.att = rope ? h->g_dk_att : nullptr;
    fk.out = dk;
    CK(hlta::launch_bwd_finalize(fk, bf16, s));
    hlta::BwdFinalizeArgs fv = fq;
    fv.acc = h->g_dv;
    fv.att = nullptr;
    fv.rope = 0;
    fv.out = dv;
    fv.d = c.d_v;
    CK(hlta::launch_bwd_finalize(fv, bf16, s));

    // gate gradients
    CK(cudaMemsetAsync(dgates, 0, (size_t)c.H * 3 * sizeof(float), s));
    for (int br = 0; br < 3; ++br)
        if (branches & (1u << br)) CK(hlta::launch_gate_grad(h->g_rowdot[br], c.B, L, c.H, br, dgates, s));
    CK(cudaGetLastError());
    return ok();
}

hlta_status hlta_forward_host(hlta_handle *h, int L, const void *q, const void *k, const void *v,
                              const float *alpha, const float *beta, const float *gates,
                              const float *S0, float *S_out, void *out, unsigned branches,
                              void *stream) {
    INJECT("hlta_forward_host");
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_forward_host: handle is NULL");
    const hlta_config &c = h->cfg;
    if (L < 1 || L > c.max_seq_len)
        return fail(HLTA_ERR_INVALID_ARG, "hlta_forward_host: L=%d outside [1, %d]", L, c.max_seq_len);
    if (!q || !k || !v || !alpha || !beta || !gates || !out)
        return fail(HLTA_ERR_INVALID_ARG, "hlta_forward_host: a required pointer is NULL");
    CK(cudaSetDevice(h->device));
    const size_t eb = h->elem_bytes;
    auto up16 = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t rows_max = (size_t)c.B * c.max_seq_len * c.H;
    const size_t nq = up16(rows_max * c.d_k * eb), nv = up16(rows_max * c.d_v * eb);
    const size_t ng = up16(rows_max * sizeof(float)), nh = up16((size_t)c.H * 3 * sizeof(float));
    const size_t ns = up16(state_elems(c) * sizeof(float));
    const size_t need = 2 * nq + 2 * nv + 2 * ng + nh + 2 * ns;
    if (!h->stage) {
        if (cudaMalloc((void **)&h->stage, need) != cudaSuccess) {
            cudaGetLastError();
            return fail(HLTA_ERR_OOM, "hlta_forward_host: staging allocation failed");
        }
        h->stage_bytes = need;
    }
    char *p = h->stage;
    void *dq = p; p += nq;
    void *dk = p; p += nq;
    void *dv = p; p += nv;
    void *dout = p; p += nv;
    float *da = (float *)p; p += ng;
    float *db = (float *)p; p += ng;
    float *dg = (float *)p; p += nh;
    float *dS0 = (float *)p; p += ns;
    float *dS1 = (float *)p;
    const size_t rows = (size_t)c.B * L * c.H;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CK(cudaMemcpyAsync(dq, q, rows * c.d_k * eb, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(dk, k, rows * c.d_k * eb, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(dv, v, rows * c.d_v * eb, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(da, alpha, rows * sizeof(float), cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(db, beta, rows * sizeof(float), cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(dg, gates, (size_t)c.H * 3 * sizeof(float), cudaMemcpyHostToDevice, s));
    if (S0) CK(cudaMemcpyAsync(dS0, S0, state_elems(c) * sizeof(float), cudaMemcpyHostToDevice, s));
    hlta_status st = hlta_forward(h, L, dq, dk, dv, da, db, dg, S0 ? dS0 : nullptr,
                                  S_out ? dS1 : nullptr, dout, branches, stream);
    if (st != HLTA_OK) return st;
    CK(cudaMemcpyAsync(out, dout, rows * c.d_v * eb, cudaMemcpyDeviceToHost, s));
    if (S_out) CK(cudaMemcpyAsync(S_out, dS1, state_elems(c) * sizeof(float), cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
    return ok();
}

hlta_status hlta_stream_step(hlta_handle *h, int n, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const float *gates, void *out,
                             unsigned branches, void *stream) {
    INJECT("hlta_stream_step");
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_step: handle is NULL");
    if (h->cfg.max_stream_tokens < 1)
        return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_step: handle created with max_stream_tokens = 0");
    if (n < 1 || n > h->cfg.max_stream_tokens)
        return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_step: n=%d outside [1, %d]", n,
                    h->cfg.max_stream_tokens);
    if (branches & ~7u) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_step: unknown branch bits");
    if (branches == 0) branches = HLTA_BRANCH_ALL;
    Inputs in{q, k, v, alpha, beta, gates};
    hlta_status st = check_inputs("hlta_stream_step", in, out);
    if (st != HLTA_OK) return st;
    CK(cudaSetDevice(h->device));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const hlta_config &c = h->cfg;
    hlta::RingAppendArgs ra;
    ra.k = k;
    ra.v = v;
    ra.ring_k = h->ring_k;
    ra.ring_v = h->ring_v;
    ra.pos0 = h->pos;
    ra.cap = h->ring_cap;
    ra.n = n;
    ra.B = c.B;
    ra.H = c.H;
    ra.d_k = c.d_k;
    ra.d_v = c.d_v;
    ra.elem_bytes = h->elem_bytes;
    CK(hlta::launch_ring_append(ra, s));
    if (h->prof) h->prof_launches += 2;
    st = run_pass(h, in, h->pos, n, h->ring_k, h->ring_v, h->ring_cap, false, h->S_stream,
                  h->S_stream, out, branches, s);
    if (st != HLTA_OK) return st;
    CK(cudaGetLastError());
    h->pos += n;
    return ok();
}

hlta_status hlta_state_get(hlta_handle *h, float *S_dst, long long *pos_out, void *stream) {
    INJECT("hlta_state_get");
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_state_get: handle is NULL");
    if (!h->S_stream) return fail(HLTA_ERR_INVALID_ARG, "hlta_state_get: streaming disabled");
    if (!S_dst) return fail(HLTA_ERR_INVALID_ARG, "hlta_state_get: S_dst is NULL");
    CK(cudaSetDevice(h->device));
    CK(cudaMemcpyAsync(S_dst, h->S_stream, state_elems(h->cfg) * sizeof(float),
                       cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
    if (pos_out) *pos_out = h->pos;
    return ok();
}

hlta_status hlta_stream_reset(hlta_handle *h, void *stream) {
    INJECT("hlta_stream_reset");
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_reset: handle is NULL");
    if (!h->S_stream) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_reset: streaming disabled");
    CK(cudaSetDevice(h->device));
    CK(cudaMemsetAsync(h->S_stream, 0, state_elems(h->cfg) * sizeof(float),
                       static_cast<cudaStream_t>(stream)));
    h->pos = 0;
    return ok();
}

long long hlta_stream_checkpoint_bytes(const hlta_handle *h) {
    if (!h || !h->S_stream) return 0;
    const hlta_config &c = h->cfg;
    return (long long)(kCkptHeader + state_elems(c) * sizeof(float) +
                       (size_t)c.B * h->ring_cap * c.H * (c.d_k + c.d_v) * h->elem_bytes);
}

hlta_status hlta_stream_save(hlta_handle *h, void *dst, void *stream) {
    INJECT("hlta_stream_save");
    if (!h || !dst) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_save: NULL argument");
    if (!h->S_stream) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_save: streaming disabled");
    CK(cudaSetDevice(h->device));
    const hlta_config &c = h->cfg;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    h->hdr[0] = kCkptMagic;
    h->hdr[1] = h->pos;
    h->hdr[2] = h->ring_cap;
    h->hdr[3] = hlta_stream_checkpoint_bytes(h);
    h->hdr[4] = ((long long)c.B << 40) ^ ((long long)c.H << 24) ^ (c.d_k << 12) ^ c.d_v;
    char *d = static_cast<char *>(dst);
    CK(cudaMemcpyAsync(d, h->hdr, sizeof h->hdr, cudaMemcpyHostToDevice, s));
    CK(cudaStreamSynchronize(s));  // hdr is pageable host memory reused by later calls
    d += kCkptHeader;
    const size_t sb = state_elems(c) * sizeof(float);
    CK(cudaMemcpyAsync(d, h->S_stream, sb, cudaMemcpyDeviceToDevice, s));
    d += sb;
    const size_t kb = (size_t)c.B * h->ring_cap * c.H * c.d_k * h->elem_bytes;
    const size_t vb = (size_t)c.B * h->ring_cap * c.H * c.d_v * h->elem_bytes;
    CK(cudaMemcpyAsync(d, h->ring_k, kb, cudaMemcpyDeviceToDevice, s));
    CK(cudaMemcpyAsync(d + kb, h->ring_v, vb, cudaMemcpyDeviceToDevice, s));
    return ok();
}

hlta_status hlta_stream_load(hlta_handle *h, const void *src, void *stream) {
    INJECT("hlta_stream_load");
    if (!h || !src) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_load: NULL argument");
    if (!h->S_stream) return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_load: streaming disabled");
    CK(cudaSetDevice(h->device));
    const hlta_config &c = h->cfg;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    long long hdr[8];
    CK(cudaMemcpyAsync(hdr, src, sizeof hdr, cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
    const long long sig = ((long long)c.B << 40) ^ ((long long)c.H << 24) ^ (c.d_k << 12) ^ c.d_v;
    if (hdr[0] != kCkptMagic || hdr[2] != h->ring_cap || hdr[3] != hlta_stream_checkpoint_bytes(h) ||
        hdr[4] != sig)
        return fail(HLTA_ERR_INVALID_ARG, "hlta_stream_load: checkpoint does not match this handle");
    const char *d = static_cast<const char *>(src) + kCkptHeader;
    const size_t sb = state_elems(c) * sizeof(float);
    CK(cudaMemcpyAsync(h->S_stream, d, sb, cudaMemcpyDeviceToDevice, s));
    d += sb;
    const size_t kb = (size_t)c.B * h->ring_cap * c.H * c.d_k * h->elem_bytes;
    const size_t vb = (size_t)c.B * h->ring_cap * c.H * c.d_v * h->elem_bytes;
    CK(cudaMemcpyAsync(h->ring_k, d, kb, cudaMemcpyDeviceToDevice, s));
    CK(cudaMemcpyAsync(h->ring_v, d + kb, vb, cudaMemcpyDeviceToDevice, s));
    h->pos = hdr[1];
    return ok();
}

hlta_status hlta_profile_enable(hlta_handle *h, int enable) {
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_profile_enable: handle is NULL");
    CK(cudaSetDevice(h->device));
    CK(cudaDeviceSynchronize());
    for (auto &m : h->marks) {
        h->event_pool.push_back(m.a);
        h->event_pool.push_back(m.b);
    }
    h->marks.clear();
    for (int i = 0; i < 3; ++i) {
        h->prof_ms[i] = 0;
        h->prof_passes[i] = 0;
    }
    h->prof_launches = 0;
    h->prof = enable != 0;
    return ok();
}

hlta_status hlta_profile_read(hlta_handle *h, hlta_profile_data *out) {
    if (!h || !out) return fail(HLTA_ERR_INVALID_ARG, "hlta_profile_read: NULL argument");
    CK(cudaSetDevice(h->device));
    CK(cudaDeviceSynchronize());
    for (auto &m : h->marks) {
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, m.a, m.b));
        h->prof_ms[m.slot] += ms;
        h->prof_passes[m.slot] += 1;
        h->event_pool.push_back(m.a);
        h->event_pool.push_back(m.b);
    }
    h->marks.clear();
    memset(out, 0, sizeof *out);
    out->count = 3;
    const char *names[3] = {"swa", "dswa", "gdn"};
    for (int i = 0; i < 3; ++i) {
        snprintf(out->name[i], sizeof out->name[i], "%s", names[i]);
        out->total_ms[i] = h->prof_ms[i];
        out->passes[i] = h->prof_passes[i];
    }
    out->kernel_launches = h->prof_launches;
    return ok();
}

hlta_status hlta_device_status(hlta_handle *h) {
    if (!h) return fail(HLTA_ERR_INVALID_ARG, "hlta_device_status: handle is NULL");
    CK(cudaSetDevice(h->device));
    CK(cudaDeviceSynchronize());
    int e = 0;
    CK(cudaMemcpy(&e, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost));
    if (e != hlta::DEVERR_NONE) {
        CK(cudaMemset(h->dev_err, 0, sizeof(int)));
        return fail(HLTA_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (code %d)", e);
    }
    return ok();
}

}  // extern "C"
