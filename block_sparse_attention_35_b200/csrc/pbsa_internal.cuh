// pbsa_internal.cuh - host-side geometry and kernel launcher declarations shared by the
// PBSA translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pbsa.h"

namespace pbsa {

// Geometry derived from a pbsa_config (all counts in tokens, blocks or frames).
// A block is bt x bh x bw tokens (sparse_kv_block_size): bt consecutive frames ("a frame
// group") x bh rows x bw columns; edge blocks are clipped to the frame.  Block ids count
// frame groups: id = group * nbf + block in group.  Every frame count the ABI takes is a
// multiple of bt.
struct Geo {
    int B, H, D;
    int fh, fw, tf;     // frame grid and tokens per frame
    int bt, bh, bw;     // block shape (frames, rows, columns)
    int brows;          // bt * bh * bw: rows of a full block (<= 64)
    int nby, nbx, nbf;  // block rows, block columns, blocks per frame group
    int W;              // frame slots of the local ring
    int Wg;             // frame groups of the ring (W / bt)
    int S;              // persistent slots (sink slots first)
    int n_sink;         // sink slots at the front of the persistent store
};

// Block i of a frame group: first row and column in the frame and its valid extent.
struct BlockBox {
    int y0, x0, hv, wv;
};

__host__ __device__ inline BlockBox block_box(const Geo& g, int i) {
    BlockBox b;
    b.y0 = g.bh * (i / g.nbx);
    b.x0 = g.bw * (i % g.nbx);
    b.hv = min(g.bh, g.fh - b.y0);
    b.wv = min(g.bw, g.fw - b.x0);
    return b;
}

// Row r (0..63) of a block as a TMA box lays it out (column fastest, then row, then frame):
// frame t, row y, column x inside the block; true when the token exists (r < brows and
// inside the frame).
__host__ __device__ inline bool block_row(const Geo& g, const BlockBox& bb, int r, int* t, int* y, int* x) {
    *x = r % g.bw;
    *y = (r / g.bw) % g.bh;
    *t = r / (g.bw * g.bh);
    return r < g.brows && *y < bb.hv && *x < bb.wv;
}

// Valid rows of block i as a 64-bit mask over its box rows (the rows block_row accepts),
// built with shifts: wv bits per row of the frame, hv rows per frame, bt frames.
__host__ __device__ inline uint64_t block_rows_mask(const Geo& g, int i) {
    const BlockBox bb = block_box(g, i);
    const uint64_t row = bb.wv >= 64 ? ~0ull : ((1ull << bb.wv) - 1ull);
    uint64_t plane = 0;
    for (int y = 0; y < bb.hv; ++y) plane |= row << (y * g.bw);
    uint64_t m = 0;
    for (int t = 0; t < g.bt; ++t) m |= plane << (t * g.bh * g.bw);
    return m;
}

// Forward-pass launch arguments.
struct FwdArgs {
    Geo g;
    int q_frames, local_frames, ring_head;
    int idx_stride;
    int ucap;            // capacity of the per-tile union of selections
    int n_seg_max;       // mass segments per CTA (S + ucap)
    const int32_t* pers_len;
    const int32_t* idx;
    const int32_t* cnt;
    float* lse;
    float* mass_local;
    float* mass_pers;
    float* scratch;      // mass partials, [ctas][n_seg_max][128]
    int32_t* status;
    CUtensorMap tm_q, tm_o, tm_kl, tm_vl, tm_kp, tm_vp;
    CUtensorMap tm_kp64, tm_vp64;  // slot store, 64-row boxes (one full slot)
};

// Backward-pass launch arguments.
struct BwdArgs {
    Geo g;
    int q_frames, local_frames, ring_head;
    int idx_stride;
    const int32_t* pers_len;
    const int32_t* idx;
    const int32_t* cnt;
    const float* lse;
    const __nv_bfloat16* out;
    const __nv_bfloat16* dout;
    float* delta;        // [B, H, Nq] workspace
    float* dq;           // zeroed by the delta pass, then accumulated by the key tiles
    float* dk_pers;
    float* dv_pers;
    float* dk_local;
    float* dv_local;
    int32_t* status;
    CUtensorMap tm_q, tm_do, tm_kl, tm_vl, tm_kp, tm_vp;
    CUtensorMap tm_kp64, tm_vp64;
    CUtensorMap tm_dq;   // dq as fp32 [B*q_frames, fh, fw, H, D], box of one block x 64 channels
};

// Launchers (return a cudaError_t from the launch).
// Pools q_frames query frames (may be 0) and the K frames in ring slots k_first.. (k_frames of
// them, mod W; may be 0); key means go to kbar by physical ring slot [B, H, W*NB_f, D].
cudaError_t launch_pool(const Geo& g, const __nv_bfloat16* q, int q_frames,
                        const __nv_bfloat16* k_local, int k_first, int k_frames,
                        float* qbar, float* kbar, cudaStream_t st);
cudaError_t launch_score_topk(const Geo& g, const float* qbar, const float* kbar, int ring_head,
                              int qb, int nl, int k, int32_t* idx, int idx_stride, int32_t* cnt,
                              float* scores, cudaStream_t st);
size_t score_topk_smem_bytes(const Geo& g, int nl);
cudaError_t launch_select_all(const Geo& g, int qb, int nl, int32_t* idx, int idx_stride, int32_t* cnt,
                              cudaStream_t st);

cudaError_t launch_attn_fwd(const FwdArgs& a, bool with_mass, cudaStream_t st);
size_t attn_fwd_smem_bytes(const Geo& g, int ucap);

cudaError_t launch_attn_bwd(const BwdArgs& a, cudaStream_t st);
size_t attn_bwd_smem_bytes(const Geo& g, int q_frames);

cudaError_t launch_cache_update(const Geo& g, const __nv_bfloat16* k_local,
                                const __nv_bfloat16* v_local, int local_frames, int ring_head,
                                float* mass_local, int n_evict_frames, int first_frame_global,
                                __nv_bfloat16* k_pers, __nv_bfloat16* v_pers, int32_t* pers_len,
                                float* pers_score, int32_t* pers_src, int32_t* upd,
                                int32_t* n_upd, cudaStream_t st);

// Appends n_frames frames (the first n_sink of them sink frames, whose first frame group is
// global group sink_group0) to the sink slots and the ring (from ring frame ring_slot on),
// pooling the ring frames' key means into kbar when it is not null.
cudaError_t launch_append(const Geo& g, const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                          int n_frames, int n_sink, int sink_group0, __nv_bfloat16* k_local,
                          __nv_bfloat16* v_local, int ring_slot, float* kbar, __nv_bfloat16* k_pers,
                          __nv_bfloat16* v_pers, int32_t* pers_len, float* pers_score,
                          int32_t* pers_src, cudaStream_t st);

cudaError_t launch_wait_selftest(int32_t* status, long long timeout_ns, cudaStream_t st);

}  // namespace pbsa

namespace pbsa {
// Shared argument handling for entry points outside pbsa_api.cu.
int api_fail(int code, const char* msg);
int api_cuda_fail(cudaError_t e, const char* what);
int api_prepare_select(const pbsa_config* cfg, const void* q, int q_frames, const void* k_local,
                       int local_frames, int ring_head, const int32_t* idx, int idx_stride,
                       const int32_t* cnt, const float* scores, Geo* geo, int* k,
                       size_t* scratch_bytes, size_t* key_offset);
}  // namespace pbsa
