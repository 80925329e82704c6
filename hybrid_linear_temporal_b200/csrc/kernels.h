// kernels.h -- launch interface between the C-ABI host code and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "hlta.h"

namespace hlta {

// How a branch kernel writes its gated output g*o into the layer output.
enum OutMode : int {
    OUT_STORE = 0,      // acc  = g*o            (fp32 workspace)
    OUT_ADD = 1,        // acc += g*o
    OUT_FINAL = 2,      // out  = acc + g*o      (cfg dtype)
    OUT_FINAL_ONLY = 3  // out  = g*o            (single selected branch)
};

// Device-side error codes written to the handle's error word.
enum DeviceError : int { DEVERR_NONE = 0, DEVERR_TIMEOUT = 1 };


// Geometry of one sliding-window branch (section 2.2.2 of the Kairos paper).
// SWA is the dilation-1 case.  Positions are absolute token indices t = f*P + s.
struct WindowGeom {
    int P;          // tokens per frame
    int dil;        // dilation (1 for SWA)
    int w;          // backward reach: keys at rearranged r' with r - w < r' (w >= 1, self included)
    int w_hi;       // forward reach: r' <= r + w_hi (0 = causal)
};

// Arguments of the SIMT attention kernel.
struct AttnSimtArgs {
    const void *q;        // [B, nq, H, d_k]; query row i has absolute position q_pos0 + i
    const void *k;        // key store [B, key_rows, H, d_k]; position p at row p % key_rows
    const void *v;        // value store [B, key_rows, H, d_v]
    long long q_pos0;
    int nq, B, H, d_k, d_v;
    long long key_rows;
    long long n_keys;     // keys exist at positions 0 .. n_keys-1 (bounds a forward reach)
    WindowGeom geom;
    float scale_log2;     // log2(e) / sqrt(d_k)
    const float *gates;   // [H, 3]
    int gate_col;         // 0 = SWA, 1 = DSWA
    int out_mode;         // OutMode
    float *acc;           // [B, nq, H, d_v] fp32
    void *out;            // [B, nq, H, d_v] dtype
};

// Arguments of the SIMT recurrent memory kernel (one token at a time).
struct GdnRecArgs {
    const void *q, *k, *v;     // [B, n, H, d]
    const float *alpha, *beta; // [B, n, H]
    const float *S_in;         // [B, H, d_v, d_k] or nullptr (zeros)
    float *S_out;              // [B, H, d_v, d_k] or nullptr; may alias S_in
    int n, B, H, d_k, d_v;
    const float *gates;
    int out_mode;
    float *acc;
    void *out;
    int form;  // HLTA_GDN_DECAYED / HLTA_GDN_PAGES: what the retrieval reads
};

struct RingAppendArgs {
    const void *k, *v;     // [B, n, H, d]
    void *ring_k, *ring_v; // [B, cap, H, d]
    long long pos0, cap;
    int n, B, H, d_k, d_v, elem_bytes;
};

// Rotary position embedding of q and k for the attention branches (a reading of
// the RoPE the pages name for the sliding-window blocks): channel pair
// (2m, 2m+1) of the token at absolute position pos0 + t is rotated by the angle
// (pos0 + t) * inv_freq[m], inv_freq[m] = base^(-2m/d).  Writes rotated copies.
struct RopeArgs {
    const void *q, *k;  // [B, n, H, d] dtype
    void *q_out, *k_out;
    int B, n, H, d;
    long long pos0;
    double inv_freq[64];
};
cudaError_t launch_rope(const RopeArgs &a, bool bf16, cudaStream_t s);

// Arguments of the CUDA-core attention backward (one branch).  q, k are the
// tensors the forward branch read (rotated copies when rotary embedding is on).
struct AttnBwdArgs {
    const void *q, *k, *v;   // [B, L, H, d] dtype
    const void *dout;        // [B, L, H, d_v] dtype: gradient of the layer output
    int L, B, H, d_k, d_v;
    WindowGeom geom;
    float scale_log2;        // log2(e) / sqrt(d_k)
    float scale;             // 1 / sqrt(d_k)
    const float *gates;      // [H, 3]
    int gate_col;            // 0 = SWA, 1 = DSWA
    float *lse;              // [B*L*H] scratch: log2-domain log-sum-exp of the row
    float *rowdot;           // [B*L*H] out: dout_i . o_i (the branch's ungated output)
    float *dq, *dk, *dv;     // [B, L, H, d] fp32 accumulators (added to)
};
cudaError_t launch_attn_bwd(const AttnBwdArgs &a, bool bf16, cudaStream_t s);

// Arguments of the chunked memory backward (gdn_bwd.cu).  Inputs [B, L, H, d]
// dtype, alpha/beta [B, L, H]; chunk-indexed scratch [B*H, nc, ...] fp32 with
// nc = ceil(L / 64); ws: grid_chunks per-CTA workspaces of ws_per_cta floats.
struct GdnBwdArgs {
    const void *q, *k, *v, *dout;
    const float *alpha, *beta, *gates;
    const float *S0;        // [B, H, d_v, d_k] or nullptr (zeros)
    const float *dS_final;  // [B, H, d_v, d_k] or nullptr (zeros)
    int L, B, H, d_k, d_v;
    float *bw_W, *bw_TbV, *bw_Kd, *bw_T, *bw_Lc, *bw_ell, *bw_S, *bw_dS, *bw_U;
    float *ws;
    size_t ws_per_cta;
    int grid_chunks;
    float *dq, *dk, *dv;    // [B, L, H, d] fp32: stored (the attention branches add after)
    float *dalpha, *dbeta;  // [B, L, H]
    float *dS0;             // [B, H, d_v, d_k] or nullptr
    float *rowdot;          // [B*L*H]: dout . o of the memory branch
};
size_t gdn_bwd_ws_floats(int d_k, int d_v);
cudaError_t launch_gdn_bwd(const GdnBwdArgs &a, bool bf16, cudaStream_t s);

// out = acc + R^T att (R: the rotary embedding when rope, else identity; att may
// be null), converted to the tensor type.  Rows are (b, t, h) with t < L.
struct BwdFinalizeArgs {
    const float *acc, *att;
    void *out;
    long long rows;
    int d, L, H;
    int rope;
    double inv_freq[64];
};
cudaError_t launch_bwd_finalize(const BwdFinalizeArgs &a, bool bf16, cudaStream_t s);
// rowdot = dout . o per row (o fp32 [B, L, H, d]), written in [B, L, H] and [B, H, L] order
cudaError_t launch_rowdot(const void *dout, const float *o, long long rows, int d, int L, int H, bool bf16,
                          float *rowdot, float *rowdot_hm, cudaStream_t s);
// dgates[h*3 + col] = sum over (b, t) of rowdot[(b*L + t)*H + h]
cudaError_t launch_gate_grad(const float *rowdot, int B, int L, int H, int col, float *dgates, cudaStream_t s);

// Sets the thread-local message returned by hlta_last_error() (empty clears it).
void set_last_error(const char *msg);

cudaError_t launch_attn_simt(const AttnSimtArgs &a, bool bf16, cudaStream_t s);
cudaError_t launch_gdn_recurrent(const GdnRecArgs &a, bool bf16, cudaStream_t s);
cudaError_t launch_ring_append(const RingAppendArgs &a, cudaStream_t s);

}  // namespace hlta
