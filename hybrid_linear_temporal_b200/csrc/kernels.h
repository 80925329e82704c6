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
    int w;          // window in (rearranged) tokens
};

// Arguments of the SIMT attention kernel.
struct AttnSimtArgs {
    const void *q;        // [B, nq, H, d_k]; query row i has absolute position q_pos0 + i
    const void *k;        // key store [B, key_rows, H, d_k]; position p at row p % key_rows
    const void *v;        // value store [B, key_rows, H, d_v]
    long long q_pos0;
    int nq, B, H, d_k, d_v;
    long long key_rows;
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

// Sets the thread-local message returned by hlta_last_error() (empty clears it).
void set_last_error(const char *msg);

cudaError_t launch_attn_simt(const AttnSimtArgs &a, bool bf16, cudaStream_t s);
cudaError_t launch_gdn_recurrent(const GdnRecArgs &a, bool bf16, cudaStream_t s);
cudaError_t launch_ring_append(const RingAppendArgs &a, cudaStream_t s);

}  // namespace hlta
