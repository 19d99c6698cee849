/*
 * pbsa.h - C ABI of the Persistent Block-Sparse Attention (PBSA) library, NVIDIA B200
 * (sm_100a).
 *
 * PBSA is the attention of "Sparse Forcing: Native Trainable Sparse Attention for
 * Real-time Autoregressive Diffusion Video Generation" (pith.science, abstract): a chunk of
 * video query tokens attends to every block of a persistent cache and to a top-k
 * selection of the token blocks (1x8x8 or 3x4x4) of a sliding local window; when the window slides,
 * the evicted blocks are merged into the persistent cache.  The argument names follow the
 * project page's usage snippet of SparseForcingAttention (boxunxu.top/SparseForcing):
 * total_cache_size, local_cache_size, persistent_cache_size, kv_cache_mode,
 * sparse_kv_block_size, max_seq_len, use_local_block_sparse_attn,
 * local_block_sparse_topk_ratio, and the call attn(query, key_persistent,
 * value_persistent, key_local, value_local).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller.  The library never
 *    allocates or frees device memory; scratch comes from the caller's `workspace`
 *    (size from pbsa_workspace_size).  Pointers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void*.  Every call is asynchronous on it and
 *    performs no host synchronisation.
 *  - Return value: PBSA_OK (0) or a negative PBSA_ERR_* code.  Argument errors are found
 *    on the host before anything is launched; pbsa_last_error() then gives a message
 *    (thread-local, valid until the next call on the same thread).
 *  - `status` (where present) is a device int32 the caller zeroes; kernels write
 *    PBSA_ERR_TIMEOUT into it when a bounded wait runs out (the kernel then returns
 *    early and its outputs are undefined) and PBSA_ERR_DEVICE_CHECK when an index read
 *    from device memory is out of range (the bad entry is skipped).
 *  - Layouts (B batch, H heads, D head dim, T_f = frame_h * frame_w tokens per frame,
 *    tokens of a frame in raster order n = y * frame_w + x, frames consecutive):
 *      query / out           [B, q_frames * T_f, H, D]      bf16
 *      key_local/value_local [B, W * T_f, H, D]              bf16, a ring of W =
 *                            local_cache_size / T_f frame slots.  The window holds
 *                            `local_frames` frames; its frame p (0 = oldest) lives in
 *                            ring slot (ring_head + p) % W.
 *      key_persistent / value_persistent [B, H, S, 64, D]   bf16: S slots of one block
 *                            each, the block's tokens in raster order in rows
 *                            0 .. pers_len-1.  Rows past pers_len never reach an output
 *                            but must hold finite values (pbsa_cache_update leaves them
 *                            zero): the kernels stream slots in 8-row groups and multiply
 *                            the masked rows by an exact zero.
 *      pers_len [B, H, S] int32 (0 = empty slot, else the block's token count, 1..64:
 *                            block_t * block_h * block_w for an interior block,
 *                            block_t * hv * wv for a block cut by the frame edge, e.g.
 *                            6 x 2 = 12 for [1,8,8] on a 30 x 50 grid).
 *  - Blocks (sparse_kv_block_size = [block_t, block_h, block_w], e.g. [1, 8, 8] or the
 *    project page's [3, 4, 4]): block_t consecutive frames (a "frame group") x block_h
 *    rows x block_w columns.  A frame group has NB = ceil(frame_h / block_h) *
 *    ceil(frame_w / block_w) blocks numbered by * ceil(frame_w / block_w) + bx; edge
 *    blocks are clipped to the frame.  Inside a block (and in a persistent slot) tokens
 *    are listed frame by frame, each frame in raster order.  Local block ids are LOGICAL:
 *    window frame group p, block i -> p * NB + i.  Query block ids: chunk frame group f,
 *    block i -> f * NB + i.  Every frame count and frame position the calls take
 *    (q_frames, local_frames, ring_head, n_evict_frames, first_frame_global, ...) must be
 *    a multiple of block_t, and so must the window (local_cache_size / T_f).
 */
#ifndef PBSA_H
#define PBSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PBSA_API __attribute__((visibility("default")))
#else
#define PBSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define PBSA_OK 0
#define PBSA_ERR_ARG (-1)          /* bad argument: null pointer, size, alignment */
#define PBSA_ERR_UNSUPPORTED (-2)  /* valid per the pages but not built here */
#define PBSA_ERR_CUDA (-3)         /* a CUDA runtime/driver call failed */
#define PBSA_ERR_TIMEOUT (-4)      /* device status: a bounded wait ran out */
#define PBSA_ERR_DEVICE_CHECK (-5) /* device status: an index was out of range */
#define PBSA_ERR_WORKSPACE (-6)    /* workspace too small */

#define PBSA_KV_CACHE_SPARSE_FORCING 0 /* kv_cache_mode="sparse_forcing" */
/* kv_cache_mode="dense" (a reading: the project page names only "sparse_forcing"; this is
 * the plain cache the pages compare against): the window is the whole total_cache_size,
 * there are no persistent slots (S = 0), every window block is attended, and a slide
 * simply drops the oldest frames.  Persistent pointers may then be NULL. */
#define PBSA_KV_CACHE_DENSE 1

/* Operation ids for pbsa_workspace_size. */
#define PBSA_OP_SELECT 0
#define PBSA_OP_FWD 1
#define PBSA_OP_BWD 2
#define PBSA_OP_UPDATE 3

/*
 * Configuration: the constructor arguments of SparseForcingAttention (project page,
 * usage snippet) plus the shapes the pages leave implicit (batch, heads, head dim and
 * the token grid of a frame).
 */
typedef struct pbsa_config {
    int B, H, D;                 /* batch, heads, head dim (64 or 128) */
    int frame_h, frame_w;        /* token grid of one frame, e.g. 30 x 52 */
    int block_t, block_h, block_w; /* sparse_kv_block_size; block_t*block_h*block_w <= 64 */
    int total_cache_size;        /* tokens; must equal local + persistent */
    int local_cache_size;        /* tokens; a whole number of frames */
    int persistent_cache_size;   /* tokens */
    int max_seq_len;             /* tokens; bounds q_frames * T_f */
    int kv_cache_mode;           /* PBSA_KV_CACHE_SPARSE_FORCING or PBSA_KV_CACHE_DENSE */
    int use_local_block_sparse_attn; /* 0: every local block is attended */
    float local_block_sparse_topk_ratio; /* in (0, 1] */
    /* Sink pattern (project page, kernel features: "local, sink, and learned top-k"; the
     * page's constructor has no such argument, this field is this library's): the first
     * sink_frames frames of a sequence (a multiple of block_t; 0 = no sink).  Their blocks
     * get slots of their own at the front of the persistent store (pbsa_sink_slots), are
     * written there by pbsa_append_frames instead of entering the window, are attended by
     * every query and are never evicted by pbsa_cache_update. */
    int sink_frames;
} pbsa_config;

/* ---------------------------------------------------------------- host-only queries */

/* Checks a configuration; PBSA_OK or an error code (message in pbsa_last_error()). */
PBSA_API int pbsa_validate_config(const pbsa_config* cfg);
/* NB, blocks per frame group (per frame when block_t = 1). */
PBSA_API int pbsa_blocks_per_frame(const pbsa_config* cfg);
/* W, frame slots of the local ring (local_cache_size / T_f; total_cache_size / T_f in
 * dense mode). */
PBSA_API int pbsa_window_frames(const pbsa_config* cfg);
/* S, persistent slots: the sink slots (pbsa_sink_slots) followed by the merged slots,
 * persistent_cache_size / (block_t * T_f) * NB when that divides, else
 * ceil(persistent_cache_size / (block_t * block_h * block_w)); 0 in dense mode. */
PBSA_API int pbsa_num_slots(const pbsa_config* cfg);
/* Sink slots at the front of the persistent store: sink_frames / block_t * NB (slot =
 * global frame group * NB + block in group). */
PBSA_API int pbsa_sink_slots(const pbsa_config* cfg);
/* k, local blocks attended per query block for a window of local_frames frames:
 * N_L = local_frames / block_t * NB; k = N_L when use_local_block_sparse_attn is 0 or in dense
 * mode, else clamp(ceil(ratio * N_L), 1, N_L).  When k = N_L and no scores are asked for,
 * pbsa_select_blocks writes the full ascending list without scoring. */
PBSA_API int pbsa_topk_count(const pbsa_config* cfg, int local_frames);
/* Workspace bytes needed by operation `op` (PBSA_OP_*) for a chunk of q_frames frames. */
PBSA_API size_t pbsa_workspace_size(const pbsa_config* cfg, int op, int q_frames);
/* Message of the last error on this thread ("" if none). */
PBSA_API const char* pbsa_last_error(void);
/* Library version string. */
PBSA_API const char* pbsa_version(void);

/* ------------------------------------------------------------------ device calls */

/*
 * Block selection: the top-k local blocks for every query block.
 * (pith.science abstract: computation inside each local window is restricted to a
 * dynamically selected neighbourhood; project page: learned top-k selection with
 * local_block_sparse_topk_ratio.)
 *
 * Score of query block b and local block j: mean of b's valid query tokens . mean of j's
 * valid key tokens / sqrt(D).  The k best (score descending, then lower logical id) are
 * written to idx[b] in ascending id order; cnt[b] = k.
 *
 *   q        [B, q_frames*T_f, H, D] bf16
 *   k_local  ring [B, W*T_f, H, D] bf16; window = local_frames frames from ring_head
 *   idx      [B, H, QB, idx_stride] int32 out (QB = q_frames / block_t * NB, idx_stride >= k)
 *   cnt      [B, H, QB] int32 out
 *   scores   nullable; [B, H, QB, N_L] fp32 out
 *   workspace >= pbsa_workspace_size(cfg, PBSA_OP_SELECT, q_frames) bytes
 */
PBSA_API int pbsa_select_blocks(const pbsa_config* cfg, const void* q, int q_frames,
                       const void* k_local, int local_frames, int ring_head,
                       int32_t* idx, int idx_stride, int32_t* cnt, float* scores,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Block selection that allocates nothing and needs no workspace.  The paper has no
 * counterpart; this is a convenience of this library.
 *
 * Some callers cannot allocate device memory where they select blocks: a plugin inside
 * an inference engine whose memory plan is fixed before it runs, or a decode loop that
 * must not call cudaMalloc because it blocks the host and synchronises the device.  This
 * call computes exactly what pbsa_select_blocks computes (same kernels, same results) but
 * keeps the pooled-mean scratch in a library-owned static device buffer of
 * PBSA_SELECT_STATIC_SCRATCH_BYTES, held by every GPU that loads the library until exit.
 *
 *  - Limit: the scratch a call needs is pbsa_workspace_size(cfg, PBSA_OP_SELECT,
 *    q_frames); above PBSA_SELECT_STATIC_SCRATCH_BYTES the call returns
 *    PBSA_ERR_UNSUPPORTED and launches nothing.
 *  - The first call on a device looks up the buffer's device address (once per device,
 *    with that device current); make that first call before any stream capture.
 *  - Every call shares the one buffer.  Calls whose kernels overlap on the GPU (different
 *    streams, or different host threads on the same device) race on it; order them on
 *    one stream or with events.  The buffer keeps the last call's contents; nothing in
 *    it needs clearing between calls.
 *  - Arguments, layouts and errors are those of pbsa_select_blocks without workspace.
 */
#define PBSA_SELECT_STATIC_SCRATCH_BYTES (8u << 20)
PBSA_API int pbsa_select_blocks_noalloc(const pbsa_config* cfg, const void* q, int q_frames,
                                        const void* k_local, int local_frames, int ring_head,
                                        int32_t* idx, int idx_stride, int32_t* cnt,
                                        float* scores, void* stream);

/*
 * Key-mean cache (project page, kernel features: the KV cache is managed by the kernels; a
 * reading, not a stated feature: a window block never changes while it is cached, so its
 * pooled key can be computed once, when its frame is appended).  The paper has no separate
 * call for this.
 *
 * pbsa_pool_keys: mean over the valid tokens of every block of the n_frames frames in ring
 * slots first_slot, first_slot+1, ... (mod W) of k_local [B, W*T_f, H, D] bf16, written to
 * kbar [B, H, (W / block_t) * NB, D] fp32 at row (slot / block_t * NB + block) - the layout
 * pbsa_select_blocks_pooled reads.  Rows of other slots are left as they are.  kbar is
 * caller-owned device memory; no workspace.  PBSA_ERR_ARG on a bad slot/frame count
 * (both multiples of block_t).
 *
 * pbsa_select_blocks_pooled: pbsa_select_blocks with the window's key means taken from kbar
 * (every slot of the window must have been pooled since its frame was written) instead of
 * being recomputed from k_local: only the chunk's queries are pooled.  Same outputs and
 * errors as pbsa_select_blocks; workspace >= B*H*QB*D*4 bytes (256-aligned),
 * not needed when every block is selected and scores is NULL.
 */
PBSA_API int pbsa_pool_keys(const pbsa_config* cfg, const void* k_local, int first_slot, int n_frames,
                            float* kbar, void* stream);
PBSA_API int pbsa_select_blocks_pooled(const pbsa_config* cfg, const void* q, int q_frames,
                                       const float* kbar, int local_frames, int ring_head,
                                       int32_t* idx, int idx_stride, int32_t* cnt, float* scores,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Frame append (the algorithm fragment: each chunk's frames enter the KV cache), fused
 * with the key-mean cache.  The paper has no separate call for this.
 *
 * k_new, v_new [B, n_frames*T_f, H, D] bf16: frames first_global_frame,
 * first_global_frame + 1, ... of the sequence (n_frames and first_global_frame multiples
 * of block_t).  Frames below cfg->sink_frames are sink frames: each of their blocks is
 * written whole into sink slot (global frame group * NB + block in group) of
 * key_persistent / value_persistent (rows past its length zeroed) with pers_len = token
 * count, pers_score = 0, pers_src = slot; sink frames come before every window frame of a
 * sequence.  Every other frame f goes to ring frame (ring_slot + f - n_sink) % W of
 * k_local / v_local, n_sink being the number of sink frames in this call
 * (clamp(sink_frames - first_global_frame, 0, n_frames)); when kbar is not NULL the mean
 * key of each of their blocks is written to kbar as pbsa_pool_keys does, in the same
 * pass.  One read of the new frames, one write of each copy.  Persistent pointers may be
 * NULL when no sink frame is appended.  ring_slot is a multiple of block_t in [0, W) and
 * the window frames appended fit in the ring (n_frames - n_sink <= W).
 */
PBSA_API int pbsa_append_frames(const pbsa_config* cfg, const void* k_new, const void* v_new,
                                int n_frames, int first_global_frame, void* k_local, void* v_local,
                                int ring_slot, float* kbar, void* k_pers, void* v_pers,
                                int32_t* pers_len, float* pers_score, int32_t* pers_src,
                                void* stream);

/*
 * PBSA forward.  (pith.science abstract; project page call attn(query, key_persistent,
 * value_persistent, key_local, value_local).)
 *
 * Each query token of query block b attends, with softmax scale 1/sqrt(D), to every valid
 * row of every occupied persistent slot and to the valid tokens of the local blocks
 * idx[b][0 .. cnt[b]).
 *
 *   out        [B, q_frames*T_f, H, D] bf16 out
 *   lse        [B, H, q_frames*T_f] fp32 out, natural-log softmax normaliser per row
 *   mass_local nullable; [B, H, (W / block_t) * NB] fp32, indexed by PHYSICAL block
 *              (ring slot / block_t * NB + block in group).  Accumulated (+=): the softmax
 *              probability summed over this chunk's query rows, per local block.
 *   mass_pers  nullable; [B, H, S] fp32, accumulated the same way per persistent slot.
 *              This is the pers_score array of pbsa_cache_update.
 *   workspace  needed only when a mass output is given:
 *              >= pbsa_workspace_size(cfg, PBSA_OP_FWD, q_frames) bytes
 *   status     device int32 (see conventions)
 */
PBSA_API int pbsa_attn_fwd(const pbsa_config* cfg, const void* q, int q_frames,
                  const void* k_pers, const void* v_pers, const int32_t* pers_len,
                  const void* k_local, const void* v_local, int local_frames, int ring_head,
                  const int32_t* idx, int idx_stride, const int32_t* cnt,
                  void* out, float* lse, float* mass_local, float* mass_pers,
                  void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/*
 * PBSA backward (project page: full gradient support for training).  Gradients of
 * sum(out * dout) with the selection idx held fixed (no gradient flows into the block
 * scores).  Inputs are the forward's inputs plus its out and lse.
 *
 *   dout      [B, q_frames*T_f, H, D] bf16
 *   dq        [B, q_frames*T_f, H, D] fp32 out (overwritten; the key tiles' shares are summed
 *             with fp32 reductions in no fixed order, so two runs agree to rounding)
 *   dk_pers, dv_pers  [B, H, S, 64, D] fp32 out; rows < pers_len overwritten, others
 *             untouched
 *   dk_local, dv_local  ring [B, W*T_f, H, D] fp32 out; tokens of the window's frames
 *             overwritten (0 where no query attended), other ring slots untouched
 *   workspace >= pbsa_workspace_size(cfg, PBSA_OP_BWD, q_frames) bytes
 */
PBSA_API int pbsa_attn_bwd(const pbsa_config* cfg, const void* q, int q_frames,
                  const void* k_pers, const void* v_pers, const int32_t* pers_len,
                  const void* k_local, const void* v_local, int local_frames, int ring_head,
                  const int32_t* idx, int idx_stride, const int32_t* cnt,
                  const void* out, const float* lse, const void* dout,
                  float* dq, float* dk_pers, float* dv_pers, float* dk_local,
                  float* dv_local, void* workspace, size_t workspace_bytes,
                  int32_t* status, void* stream);

/*
 * Window slide and persistent merge (pith.science abstract: persistent blocks are
 * compressed, preserved and updated; algorithm fragment: the t=0 pass updates P and L).
 *
 * The oldest n_evict_frames frames of the window leave it.  The sink slots take no part.
 * Candidates are the occupied merged slots (score pers_score) followed by the evicted blocks in logical id order (score
 * mass_local of their physical block).  Ordered by score descending, ties by that
 * candidate order, the first min(S - sink slots, #candidates) are kept.  Kept slots stay in place;
 * the free slots (empty ones ascending, then dropped ones ascending) receive the kept
 * evicted blocks in id order: tokens copied frame by frame in raster order, pers_len =
 * token count, pers_score = the block's mass, pers_src = global frame group * NB + block
 * in group (global frame group = global frame / block_t), where the oldest window frame
 * has global number first_frame_global.  Dropped slots that
 * receive nothing become empty (len 0, score 0, src -1).  The evicted blocks'
 * mass_local entries are reset to 0.  The caller then advances its ring:
 * ring_head = (ring_head + n_evict_frames) % W, local_frames -= n_evict_frames.
 *
 *   upd    [B, H, n_evict_frames / block_t * NB, 2] int32 out: (slot, logical block id) per
 *          admission, in admission order
 *   n_upd  [B, H] int32 out: admissions per (b, h)
 *   workspace >= pbsa_workspace_size(cfg, PBSA_OP_UPDATE, 0) bytes
 */
PBSA_API int pbsa_cache_update(const pbsa_config* cfg, const void* k_local, const void* v_local,
                      int local_frames, int ring_head, float* mass_local,
                      int n_evict_frames, int first_frame_global,
                      void* k_pers, void* v_pers, int32_t* pers_len, float* pers_score,
                      int32_t* pers_src, int32_t* upd, int32_t* n_upd,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Diagnostic: runs one kernel that waits, with the library's bounded wait, on a barrier
 * that nothing completes.  After `timeout_ns` nanoseconds the wait gives up and writes
 * PBSA_ERR_TIMEOUT into *status.  The pages have no counterpart; it exists so that the
 * timeout path can be tested without hanging a GPU.
 */
PBSA_API int pbsa_wait_selftest(int32_t* status, long long timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PBSA_H */
