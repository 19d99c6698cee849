// pbsa_api.cu - the C ABI of include/pbsa.h: argument checks, geometry, TMA descriptors
// and kernel launches.  Nothing here allocates device memory or synchronises the host.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "pbsa.h"
#include "pbsa_internal.cuh"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(PBSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int tokens_per_frame(const pbsa_config* c) { return c->frame_h * c->frame_w; }

// blocks of one frame group (block_t frames)
int blocks_per_frame(const pbsa_config* c) {
    return ((c->frame_h + c->block_h - 1) / c->block_h) * ((c->frame_w + c->block_w - 1) / c->block_w);
}

bool dense_mode(const pbsa_config* c) { return c->kv_cache_mode == PBSA_KV_CACHE_DENSE; }

// tokens of the local ring: the local cache, or the whole cache in dense mode
int window_tokens(const pbsa_config* c) { return dense_mode(c) ? c->total_cache_size : c->local_cache_size; }

int sink_slot_count(const pbsa_config* c) {
    return dense_mode(c) ? 0 : c->sink_frames / c->block_t * blocks_per_frame(c);
}

// sink slots, then the slots of persistent_cache_size
int num_slots(const pbsa_config* c) {
    if (dense_mode(c)) return 0;
    const int n_sink = sink_slot_count(c);
    const int tg = tokens_per_frame(c) * c->block_t;
    if (c->persistent_cache_size % tg == 0) return n_sink + c->persistent_cache_size / tg * blocks_per_frame(c);
    const int brows = c->block_t * c->block_h * c->block_w;
    return n_sink + (c->persistent_cache_size + brows - 1) / brows;
}

int topk_count(const pbsa_config* c, int local_frames) {
    const int nl = local_frames / c->block_t * blocks_per_frame(c);
    if (nl <= 0) return 0;
    if (!c->use_local_block_sparse_attn || dense_mode(c)) return nl;
    const double k = std::ceil(static_cast<double>(c->local_block_sparse_topk_ratio) * nl);
    int ki = static_cast<int>(k);
    if (ki < 1) ki = 1;
    if (ki > nl) ki = nl;
    return ki;
}

int validate(const pbsa_config* c) {
    if (!c) return fail(PBSA_ERR_ARG, "config is NULL");
    if (c->B < 1 || c->H < 1) return fail(PBSA_ERR_ARG, "B and H must be >= 1 (B=%d H=%d)", c->B, c->H);
    if (c->B > 65535 || c->H > 65535) return fail(PBSA_ERR_ARG, "B and H must be <= 65535");
    if (c->D != 64 && c->D != 128) return fail(PBSA_ERR_UNSUPPORTED, "head dim %d: only 64 and 128 are built", c->D);
    if (c->H * c->D > 8192) return fail(PBSA_ERR_UNSUPPORTED, "H*D = %d > 8192", c->H * c->D);
    if (c->frame_h < 1 || c->frame_w < 1) return fail(PBSA_ERR_ARG, "frame grid %dx%d", c->frame_h, c->frame_w);
    if (c->block_t < 1 || c->block_h < 1 || c->block_w < 1)
        return fail(PBSA_ERR_ARG, "sparse_kv_block_size [%d,%d,%d]: sizes must be >= 1", c->block_t,
                    c->block_h, c->block_w);
    if (c->block_t * c->block_h * c->block_w > 64)
        return fail(PBSA_ERR_UNSUPPORTED, "sparse_kv_block_size [%d,%d,%d]: blocks above 64 tokens are not built",
                    c->block_t, c->block_h, c->block_w);
    if (c->kv_cache_mode != PBSA_KV_CACHE_SPARSE_FORCING && c->kv_cache_mode != PBSA_KV_CACHE_DENSE)
        return fail(PBSA_ERR_UNSUPPORTED, "kv_cache_mode %d: only sparse_forcing and dense are built",
                    c->kv_cache_mode);
    const int tf = tokens_per_frame(c);
    const int tg = tf * c->block_t;   // a frame group: the frames one block spans
    if (c->local_cache_size < tg || c->local_cache_size % tg)
        return fail(PBSA_ERR_ARG, "local_cache_size %d is not a positive multiple of %d tokens (%d frame(s))",
                    c->local_cache_size, tg, c->block_t);
    if (dense_mode(c) && c->total_cache_size % tg)
        return fail(PBSA_ERR_ARG, "dense mode: total_cache_size %d is not a multiple of %d tokens",
                    c->total_cache_size, tg);
    if (c->persistent_cache_size < 0) return fail(PBSA_ERR_ARG, "persistent_cache_size < 0");
    if (c->total_cache_size != c->local_cache_size + c->persistent_cache_size)
        return fail(PBSA_ERR_ARG, "total_cache_size %d != local %d + persistent %d",
                    c->total_cache_size, c->local_cache_size, c->persistent_cache_size);
    if (c->max_seq_len < tg) return fail(PBSA_ERR_ARG, "max_seq_len %d < one frame group (%d)", c->max_seq_len, tg);
    const float r = c->local_block_sparse_topk_ratio;
    if (!(r > 0.f && r <= 1.f)) return fail(PBSA_ERR_ARG, "local_block_sparse_topk_ratio %g not in (0, 1]", r);
    if (c->sink_frames < 0 || c->sink_frames % c->block_t)
        return fail(PBSA_ERR_ARG, "sink_frames %d is not a non-negative multiple of block_t %d", c->sink_frames,
                    c->block_t);
    if (c->sink_frames > 0 && dense_mode(c))
        return fail(PBSA_ERR_UNSUPPORTED, "sink frames in kv_cache_mode=dense are not built");
    const int W = window_tokens(c) / tf;
    const int nlmax = W / c->block_t * blocks_per_frame(c);
    if (nlmax > 512) return fail(PBSA_ERR_UNSUPPORTED, "%d local blocks > 512", nlmax);
    if (num_slots(c) > 1024) return fail(PBSA_ERR_UNSUPPORTED, "%d persistent slots > 1024", num_slots(c));
    return PBSA_OK;
}

pbsa::Geo make_geo(const pbsa_config* c) {
    pbsa::Geo g;
    g.B = c->B;
    g.H = c->H;
    g.D = c->D;
    g.fh = c->frame_h;
    g.fw = c->frame_w;
    g.tf = c->frame_h * c->frame_w;
    g.bt = c->block_t;
    g.bh = c->block_h;
    g.bw = c->block_w;
    g.brows = g.bt * g.bh * g.bw;
    g.nby = (c->frame_h + g.bh - 1) / g.bh;
    g.nbx = (c->frame_w + g.bw - 1) / g.bw;
    g.nbf = g.nby * g.nbx;
    g.W = window_tokens(c) / g.tf;
    g.Wg = g.W / g.bt;
    g.S = num_slots(c);
    g.n_sink = sink_slot_count(c);
    return g;
}

int check_window(const pbsa_config* c, const pbsa::Geo& g, int q_frames, int local_frames, int ring_head) {
    if (q_frames < 1) return fail(PBSA_ERR_ARG, "q_frames %d < 1", q_frames);
    if ((long long)q_frames * g.tf > c->max_seq_len)
        return fail(PBSA_ERR_ARG, "q_frames*T_f = %lld > max_seq_len %d", (long long)q_frames * g.tf, c->max_seq_len);
    // an empty window is allowed: a chunk made only of sink frames attends the slots alone
    if (local_frames < 0 || local_frames > g.W)
        return fail(PBSA_ERR_ARG, "local_frames %d not in [0, %d]", local_frames, g.W);
    if (ring_head < 0 || ring_head >= g.W) return fail(PBSA_ERR_ARG, "ring_head %d not in [0, %d)", ring_head, g.W);
    if (q_frames % g.bt || local_frames % g.bt || ring_head % g.bt)
        return fail(PBSA_ERR_ARG, "q_frames %d, local_frames %d and ring_head %d must be multiples of block_t %d",
                    q_frames, local_frames, ring_head, g.bt);
    return PBSA_OK;
}

#define REQUIRE_PTR(p)                                                        \
    do {                                                                      \
        if (!(p)) return fail(PBSA_ERR_ARG, "%s is NULL", #p);                \
        if (!aligned16(p)) return fail(PBSA_ERR_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)

#define OPTIONAL_PTR(p)                                                       \
    do {                                                                      \
        if ((p) && !aligned16(p)) return fail(PBSA_ERR_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)

// persistent-cache arguments: required when there are slots, ignored (may be NULL) when S = 0
#define PERS_PTR(g, p)                                                        \
    do {                                                                      \
        if ((g).S > 0) REQUIRE_PTR(p);                                        \
    } while (0)

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [frames, frame_h, frame_w, H, D] bf16 tensor, box [bt, bh, bw, 1, 64] (one block, its rows
// in frame / row / column order), 128-byte swizzle.
int map_tokens(CUtensorMap* m, const void* ptr, const pbsa::Geo& g, long long frames) {
    auto enc = encode_fn();
    if (!enc) return fail(PBSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.H, (cuuint64_t)g.fw, (cuuint64_t)g.fh,
                          (cuuint64_t)frames};
    cuuint64_t strides[4] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.H * g.D * 2,
                             (cuuint64_t)g.fw * g.H * g.D * 2, (cuuint64_t)g.fh * g.fw * g.H * g.D * 2};
    cuuint32_t box[5] = {64, 1, (cuuint32_t)g.bw, (cuuint32_t)g.bh, (cuuint32_t)g.bt};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBSA_ERR_CUDA, "cuTensorMapEncodeTiled (tokens) failed: %d", (int)r);
    return PBSA_OK;
}

// The same token layout as map_tokens for an fp32 tensor, unswizzled: one box is a block's
// rows x 64 channels, 256 bytes per row (the backward adds dQ tiles through it).
int map_tokens_f32(CUtensorMap* m, const void* ptr, const pbsa::Geo& g, long long frames) {
    auto enc = encode_fn();
    if (!enc) return fail(PBSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.H, (cuuint64_t)g.fw, (cuuint64_t)g.fh,
                          (cuuint64_t)frames};
    cuuint64_t strides[4] = {(cuuint64_t)g.D * 4, (cuuint64_t)g.H * g.D * 4,
                             (cuuint64_t)g.fw * g.H * g.D * 4, (cuuint64_t)g.fh * g.fw * g.H * g.D * 4};
    cuuint32_t box[5] = {64, 1, (cuuint32_t)g.bw, (cuuint32_t)g.bh, (cuuint32_t)g.bt};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<void*>(ptr), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBSA_ERR_CUDA, "cuTensorMapEncodeTiled (fp32 tokens) failed: %d", (int)r);
    return PBSA_OK;
}

// [rows, D] bf16 tensor (persistent slots, 64 rows each), box [8, 64], 128-byte swizzle.
int map_rows(CUtensorMap* m, const void* ptr, const pbsa::Geo& g, long long rows, int box_rows = 8) {
    auto enc = encode_fn();
    if (!enc) return fail(PBSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[2] = {(cuuint64_t)g.D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)g.D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PBSA_ERR_CUDA, "cuTensorMapEncodeTiled (rows) failed: %d", (int)r);
    return PBSA_OK;
}

// The two slot-store maps (8-row and 64-row boxes).  With no slots the kernels never load
// from them; they are then encoded over the window buffer so that every map is valid.
int map_slots(CUtensorMap* m8, CUtensorMap* m64, const void* pers, const void* window, const pbsa::Geo& g) {
    long long rows = (long long)g.B * g.H * g.S * 64;
    const void* base = pers;
    if (g.S == 0) {
        rows = (long long)g.B * g.W * g.tf * g.H;
        base = window;
    }
    int rc = map_rows(m8, base, g, rows, rows < 8 ? (int)rows : 8);
    if (rc != PBSA_OK) return rc;
    return map_rows(m64, base, g, rows, rows < 64 ? (int)rows : 64);
}

size_t select_ws(const pbsa::Geo& g, int q_frames) {
    return align256(sizeof(float) * (size_t)g.B * g.H * (q_frames / g.bt) * g.nbf * g.D) +
           align256(sizeof(float) * (size_t)g.B * g.H * g.Wg * g.nbf * g.D);
}

int fwd_ucap(const pbsa_config* c, const pbsa::Geo& g, int idx_stride) {
    const int kmax = topk_count(c, g.W);
    return 2 * (idx_stride < kmax ? idx_stride : kmax);
}

size_t fwd_ws(const pbsa_config* c, const pbsa::Geo& g, int q_frames) {
    // per CTA of four query blocks, two 128-row sides
    const size_t ctas = (size_t)g.B * g.H * 2 * ((q_frames / g.bt * g.nbf + 3) / 4);
    const size_t nseg = (size_t)g.S + 2 * topk_count(c, g.W);
    return align256(sizeof(float) * ctas * nseg * 128);
}

size_t bwd_ws(const pbsa::Geo& g, int q_frames) {
    return align256(sizeof(float) * (size_t)g.B * g.H * q_frames * g.tf);
}

}  // namespace

extern "C" {

const char* pbsa_last_error(void) { return g_err.c_str(); }

const char* pbsa_version(void) { return "pbsa-b200 0.1 (sm_100a)"; }

int pbsa_validate_config(const pbsa_config* cfg) { return validate(cfg); }

int pbsa_blocks_per_frame(const pbsa_config* cfg) {
    if (validate(cfg) != PBSA_OK) return -1;
    return blocks_per_frame(cfg);
}

int pbsa_window_frames(const pbsa_config* cfg) {
    if (validate(cfg) != PBSA_OK) return -1;
    return window_tokens(cfg) / tokens_per_frame(cfg);
}

int pbsa_num_slots(const pbsa_config* cfg) {
    if (validate(cfg) != PBSA_OK) return -1;
    return num_slots(cfg);
}

int pbsa_sink_slots(const pbsa_config* cfg) {
    if (validate(cfg) != PBSA_OK) return -1;
    return sink_slot_count(cfg);
}

int pbsa_topk_count(const pbsa_config* cfg, int local_frames) {
    if (validate(cfg) != PBSA_OK) return -1;
    if (local_frames < 0 || local_frames > window_tokens(cfg) / tokens_per_frame(cfg))
        return fail(PBSA_ERR_ARG, "local_frames %d out of range", local_frames);
    return topk_count(cfg, local_frames);
}

size_t pbsa_workspace_size(const pbsa_config* cfg, int op, int q_frames) {
    if (validate(cfg) != PBSA_OK) return 0;
    const pbsa::Geo g = make_geo(cfg);
    switch (op) {
        case PBSA_OP_SELECT: return select_ws(g, q_frames);
        case PBSA_OP_FWD: return fwd_ws(cfg, g, q_frames);
        case PBSA_OP_BWD: return bwd_ws(g, q_frames);
        case PBSA_OP_UPDATE: return 0;
        default: fail(PBSA_ERR_ARG, "unknown op %d", op); return 0;
    }
}

int pbsa_select_blocks(const pbsa_config* cfg, const void* q, int q_frames, const void* k_local,
                       int local_frames, int ring_head, int32_t* idx, int idx_stride, int32_t* cnt,
                       float* scores, void* workspace, size_t workspace_bytes, void* stream) {
    pbsa::Geo g;
    int k = 0;
    size_t need = 0, key_off = 0;
    int rc = pbsa::api_prepare_select(cfg, q, q_frames, k_local, local_frames, ring_head, idx, idx_stride,
                                      cnt, scores, &g, &k, &need, &key_off);
    if (rc != PBSA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int qb = q_frames / g.bt * g.nbf, nl = local_frames / g.bt * g.nbf;
    if (k == nl && !scores) {   // every window block, no scores: no pooling, no workspace
        cudaError_t e = pbsa::launch_select_all(g, qb, nl, idx, idx_stride, cnt, st);
        if (e != cudaSuccess) return cuda_fail(e, "select-all kernel launch");
        return PBSA_OK;
    }
    REQUIRE_PTR(workspace);
    if (workspace_bytes < need) return fail(PBSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
    float* qbar = static_cast<float*>(workspace);
    float* kbar = reinterpret_cast<float*>(static_cast<char*>(workspace) + key_off);
    cudaError_t e = pbsa::launch_pool(g, static_cast<const __nv_bfloat16*>(q), q_frames,
                                      static_cast<const __nv_bfloat16*>(k_local), ring_head, local_frames,
                                      qbar, kbar, st);
    if (e != cudaSuccess) return cuda_fail(e, "pool kernel launch");
    e = pbsa::launch_score_topk(g, qbar, kbar, ring_head, qb, nl, k, idx, idx_stride, cnt, scores, st);
    if (e != cudaSuccess) return cuda_fail(e, "score/top-k kernel launch");
    return PBSA_OK;
}

int pbsa_append_frames(const pbsa_config* cfg, const void* k_new, const void* v_new, int n_frames,
                       int first_global_frame, void* k_local, void* v_local, int ring_slot, float* kbar,
                       void* k_pers, void* v_pers, int32_t* pers_len, float* pers_score, int32_t* pers_src,
                       void* stream) {
    int rc = validate(cfg);
    if (rc != PBSA_OK) return rc;
    const pbsa::Geo g = make_geo(cfg);
    if (n_frames < 0 || n_frames % g.bt) return fail(PBSA_ERR_ARG, "n_frames %d is not a multiple of block_t %d", n_frames, g.bt);
    if (first_global_frame < 0 || first_global_frame % g.bt)
        return fail(PBSA_ERR_ARG, "first_global_frame %d is not a non-negative multiple of block_t %d",
                    first_global_frame, g.bt);
    if (ring_slot < 0 || ring_slot >= g.W || ring_slot % g.bt)
        return fail(PBSA_ERR_ARG, "ring_slot %d is not a multiple of block_t in [0, %d)", ring_slot, g.W);
    int n_sink = cfg->sink_frames - first_global_frame;
    n_sink = n_sink < 0 ? 0 : (n_sink > n_frames ? n_frames : n_sink);
    if (n_frames - n_sink > g.W) return fail(PBSA_ERR_ARG, "%d window frames do not fit a ring of %d", n_frames - n_sink, g.W);
    if (n_frames == 0) return PBSA_OK;
    REQUIRE_PTR(k_new);
    REQUIRE_PTR(v_new);
    if (n_frames > n_sink) {
        REQUIRE_PTR(k_local);
        REQUIRE_PTR(v_local);
        OPTIONAL_PTR(kbar);
    }
    if (n_sink > 0) {
        REQUIRE_PTR(k_pers);
        REQUIRE_PTR(v_pers);
        REQUIRE_PTR(pers_len);
        REQUIRE_PTR(pers_score);
        REQUIRE_PTR(pers_src);
    }
    cudaError_t e = pbsa::launch_append(
        g, static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new), n_frames, n_sink,
        first_global_frame / g.bt, static_cast<__nv_bfloat16*>(k_local), static_cast<__nv_bfloat16*>(v_local),
        ring_slot, kbar, static_cast<__nv_bfloat16*>(k_pers), static_cast<__nv_bfloat16*>(v_pers), pers_len,
        pers_score, pers_src, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
    return PBSA_OK;
}

int pbsa_pool_keys(const pbsa_config* cfg, const void* k_local, int first_slot, int n_frames, float* kbar,
                   void* stream) {
    int rc = validate(cfg);
    if (rc != PBSA_OK) return rc;
    const pbsa::Geo g = make_geo(cfg);
    if (first_slot < 0 || first_slot >= g.W) return fail(PBSA_ERR_ARG, "first_slot %d not in [0, %d)", first_slot, g.W);
    if (n_frames < 0 || n_frames > g.W) return fail(PBSA_ERR_ARG, "n_frames %d not in [0, %d]", n_frames, g.W);
    if (first_slot % g.bt || n_frames % g.bt)
        return fail(PBSA_ERR_ARG, "first_slot %d and n_frames %d must be multiples of block_t %d", first_slot,
                    n_frames, g.bt);
    REQUIRE_PTR(k_local);
    REQUIRE_PTR(kbar);
    cudaError_t e = pbsa::launch_pool(g, nullptr, 0, static_cast<const __nv_bfloat16*>(k_local), first_slot,
                                      n_frames, nullptr, kbar, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pool kernel launch");
    return PBSA_OK;
}

int pbsa_select_blocks_pooled(const pbsa_config* cfg, const void* q, int q_frames, const float* kbar,
                              int local_frames, int ring_head, int32_t* idx, int idx_stride, int32_t* cnt,
                              float* scores, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = validate(cfg);
    if (rc != PBSA_OK) return rc;
    const pbsa::Geo g = make_geo(cfg);
    if ((rc = check_window(cfg, g, q_frames, local_frames, ring_head)) != PBSA_OK) return rc;
    REQUIRE_PTR(q);
    REQUIRE_PTR(kbar);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(cnt);
    OPTIONAL_PTR(scores);
    const int k = topk_count(cfg, local_frames);
    if (idx_stride < k) return fail(PBSA_ERR_ARG, "idx_stride %d < k %d", idx_stride, k);
    const int nl = local_frames / g.bt * g.nbf;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (k == nl && !scores) {
        cudaError_t e = pbsa::launch_select_all(g, q_frames / g.bt * g.nbf, nl, idx, idx_stride, cnt, st);
        if (e != cudaSuccess) return cuda_fail(e, "select-all kernel launch");
        return PBSA_OK;
    }
    REQUIRE_PTR(workspace);
    const size_t need = align256(sizeof(float) * (size_t)g.B * g.H * (q_frames / g.bt) * g.nbf * g.D);
    if (workspace_bytes < need) return fail(PBSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
    if (pbsa::score_topk_smem_bytes(g, nl) > 227 * 1024)
        return fail(PBSA_ERR_UNSUPPORTED, "%d local blocks do not fit the scoring kernel", nl);
    float* qbar = static_cast<float*>(workspace);
    cudaError_t e = pbsa::launch_pool(g, static_cast<const __nv_bfloat16*>(q), q_frames, nullptr, 0, 0, qbar,
                                      nullptr, st);
    if (e != cudaSuccess) return cuda_fail(e, "pool kernel launch");
    e = pbsa::launch_score_topk(g, qbar, kbar, ring_head, q_frames / g.bt * g.nbf, nl, k, idx, idx_stride, cnt, scores, st);
    if (e != cudaSuccess) return cuda_fail(e, "score/top-k kernel launch");
    return PBSA_OK;
}

int pbsa_attn_fwd(const pbsa_config* cfg, const void* q, int q_frames, const void* k_pers,
                  const void* v_pers, const int32_t* pers_len, const void* k_local, const void* v_local,
                  int local_frames, int ring_head, const int32_t* idx, int idx_stride, const int32_t* cnt,
                  void* out, float* lse, float* mass_local, float* mass_pers, void* workspace,
                  size_t workspace_bytes, int32_t* status, void* stream) {
    int rc = validate(cfg);
    if (rc != PBSA_OK) return rc;
    const pbsa::Geo g = make_geo(cfg);
    if ((rc = check_window(cfg, g, q_frames, local_frames, ring_head)) != PBSA_OK) return rc;
    REQUIRE_PTR(q);
    PERS_PTR(g, k_pers);
    PERS_PTR(g, v_pers);
    PERS_PTR(g, pers_len);
    REQUIRE_PTR(k_local);
    REQUIRE_PTR(v_local);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(cnt);
    REQUIRE_PTR(out);
    REQUIRE_PTR(lse);
    REQUIRE_PTR(status);
    OPTIONAL_PTR(mass_local);
    OPTIONAL_PTR(mass_pers);
    if (idx_stride < 1) return fail(PBSA_ERR_ARG, "idx_stride %d < 1", idx_stride);
    const bool with_mass = mass_local || mass_pers;
    if (with_mass) {
        REQUIRE_PTR(workspace);
        const size_t need = fwd_ws(cfg, g, q_frames);
        if (workspace_bytes < need)
            return fail(PBSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
    }
    pbsa::FwdArgs a;
    a.g = g;
    a.q_frames = q_frames;
    a.local_frames = local_frames;
    a.ring_head = ring_head;
    a.idx_stride = idx_stride;
    a.ucap = fwd_ucap(cfg, g, idx_stride);
    a.n_seg_max = g.S + 2 * topk_count(cfg, g.W);
    a.pers_len = pers_len;
    a.idx = idx;
    a.cnt = cnt;
    a.lse = lse;
    a.mass_local = mass_local;
    a.mass_pers = mass_pers;
    a.scratch = static_cast<float*>(workspace);
    a.status = status;
    if (pbsa::attn_fwd_smem_bytes(g, a.ucap) > 227 * 1024)
        return fail(PBSA_ERR_UNSUPPORTED, "forward tables do not fit in shared memory");
    if ((rc = map_tokens(&a.tm_q, q, g, (long long)g.B * q_frames)) != PBSA_OK) return rc;
    if ((rc = map_tokens(&a.tm_o, out, g, (long long)g.B * q_frames)) != PBSA_OK) return rc;
    if ((rc = map_tokens(&a.tm_kl, k_local, g, (long long)g.B * g.W)) != PBSA_OK) return rc;
    if ((rc = map_tokens(&a.tm_vl, v_local, g, (long long)g.B * g.W)) != PBSA_OK) return rc;
    if ((rc = map_slots(&a.tm_kp, &a.tm_kp64, k_pers, k_local, g)) != PBSA_OK) return rc;
    if ((rc = map_slots(&a.tm_vp, &a.tm_vp64, v_pers, v_local, g)) != PBSA_OK) return rc;
    cudaError_t e = pbsa::launch_attn_fwd(a, with_mass, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "forward kernel launch");
    return PBSA_OK;
}

int pbsa_attn_bwd(const pbsa_config* cfg, const void* q, int q_frames, const void* k_pers,
                  const void* v_pers, const int32_t* pers_len, const void* k_local, const void* v_local,
                  int local_frames, int ring_head, const int32_t* idx, int idx_stride, const int32_t* cnt,
                  const void* out, const float* lse, const void* dout, float* dq, float* dk_pers,
                  float* dv_pers, float* dk_local, float* dv_local, void* workspace,
                  size_t workspace_bytes, int32_t* status, void* stream) {
    int rc = validate(cfg);
    if (rc != PBSA_OK) return rc;
    const pbsa::Geo g = make_geo(cfg);
    if ((rc = check_window(cfg, g, q_frames, local_frames, ring_head)) != PBSA_OK) return rc;
    REQUIRE_PTR(q);
    PERS_PTR(g, k_pers);
    PERS_PTR(g, v_pers);
    PERS_PTR(g, pers_len);
    REQUIRE_PTR(k_local);
    REQUIRE_PTR(v_local);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(cnt);
    REQUIRE_PTR(out);
    REQUIRE_PTR(lse);
    REQUIRE_PTR(dout);
    REQUIRE_PTR(dq);
    PERS_PTR(g, dk_pers);
    PERS_PTR(g, dv_pers);
    REQUIRE_PTR(dk_local);
    REQUIRE_PTR(dv_local);
    REQUIRE_PTR(workspace);
    REQUIRE_PTR(status);
    if (idx_stride < 1) return fail(PBSA_ERR_ARG, "idx_stride %d < 1", idx_stride);
    const size_t need = bwd_ws(g, q_frames);
    if (workspace_bytes < need) return fail(PBSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", workspace_bytes, need);
    pbsa::BwdArgs a;
    a.g = g;
    a.q_frames = q_frames;
    a.local_frames = local_frames;
    a.ring_head = ring_head;
    a.idx_stride = idx_stride;
    a.pers_len = pers_len;
    a.idx = idx;
    a.cnt = cnt;
    a.lse = lse;
    a.out = static_cast<const __nv_bfloat16*>(out);
    a.dout = static_cast<const __nv_bfloat16*>(dout);
    a.delta = static_cast<float*>(workspace);
    a.dq = dq;
    a.dk_pers = dk_pers;
    a.dv_pers = dv_pers;
    a.dk_local = dk_local;
    a.dv_local = dv_local;
    a.status = status;
    if (pbsa::attn_bwd_smem_bytes(g, q_frames) > 227 * 1024)
        return fail(PBSA_ERR_UNSUPPORTED, "backward tables do not fit in shared memory");
    if ((rc = map_tokens(&a.tm_q, q, g, (long long)g.B * q_frames)) != PBSA_OK) return rc;
    if ((rc = map_tokens(&a.tm_do, dout, g, (long long)g.B * q_frames)) != PBSA_OK) return rc;
    if ((rc = map_tokens_f32(&a.tm_dq, dq, g, (long long)g.B * q_frames)) != PBSA_OK) return rc;
    if ((rc = map_tokens(&a.tm_kl, k_local, g, (long long)g.B * g.W)) != PBSA_OK) return rc;
    if ((rc = map_tokens(&a.tm_vl, v_local, g, (long long)g.B * g.W)) != PBSA_OK) return rc;
    if ((rc = map_slots(&a.tm_kp, &a.tm_kp64, k_pers, k_local, g)) != PBSA_OK) return rc;
    if ((rc = map_slots(&a.tm_vp, &a.tm_vp64, v_pers, v_local, g)) != PBSA_OK) return rc;
    cudaError_t e = pbsa::launch_attn_bwd(a, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return fail(PBSA_ERR_UNSUPPORTED, "backward kernel not built");
    if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
    return PBSA_OK;
}

int pbsa_cache_update(const pbsa_config* cfg, const void* k_local, const void* v_local, int local_frames,
                      int ring_head, float* mass_local, int n_evict_frames, int first_frame_global,
                      void* k_pers, void* v_pers, int32_t* pers_len, float* pers_score, int32_t* pers_src,
                      int32_t* upd, int32_t* n_upd, void* workspace, size_t workspace_bytes, void* stream) {
    (void)workspace;
    (void)workspace_bytes;
    int rc = validate(cfg);
    if (rc != PBSA_OK) return rc;
    const pbsa::Geo g = make_geo(cfg);
    if ((rc = check_window(cfg, g, g.bt, local_frames, ring_head)) != PBSA_OK) return rc;
    if (n_evict_frames < 0 || n_evict_frames > local_frames)
        return fail(PBSA_ERR_ARG, "n_evict_frames %d not in [0, local_frames=%d]", n_evict_frames, local_frames);
    if (first_frame_global < 0) return fail(PBSA_ERR_ARG, "first_frame_global < 0");
    if (n_evict_frames % g.bt || first_frame_global % g.bt)
        return fail(PBSA_ERR_ARG, "n_evict_frames %d and first_frame_global %d must be multiples of block_t %d",
                    n_evict_frames, first_frame_global, g.bt);
    REQUIRE_PTR(k_local);
    REQUIRE_PTR(v_local);
    REQUIRE_PTR(mass_local);
    PERS_PTR(g, k_pers);
    PERS_PTR(g, v_pers);
    PERS_PTR(g, pers_len);
    PERS_PTR(g, pers_score);
    PERS_PTR(g, pers_src);
    REQUIRE_PTR(upd);
    REQUIRE_PTR(n_upd);
    cudaError_t e = pbsa::launch_cache_update(
        g, static_cast<const __nv_bfloat16*>(k_local), static_cast<const __nv_bfloat16*>(v_local), local_frames,
        ring_head, mass_local, n_evict_frames, first_frame_global, static_cast<__nv_bfloat16*>(k_pers),
        static_cast<__nv_bfloat16*>(v_pers), pers_len, pers_score, pers_src, upd, n_upd,
        static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cache update kernel launch");
    return PBSA_OK;
}

int pbsa_wait_selftest(int32_t* status, long long timeout_ns, void* stream) {
    REQUIRE_PTR(status);
    if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return fail(PBSA_ERR_ARG, "timeout_ns out of (0, 10 s]");
    cudaError_t e = pbsa::launch_wait_selftest(status, timeout_ns, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
    return PBSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// Helpers for entry points defined in other translation units.
namespace pbsa {

int api_fail(int code, const char* msg) { return fail(code, "%s", msg); }

int api_cuda_fail(cudaError_t e, const char* what) { return cuda_fail(e, what); }

// Checks the arguments of a block selection call exactly as pbsa_select_blocks does and
// returns the geometry, k, and the bytes of pooled-mean scratch the call needs (query
// means first, key means at key_offset).
int api_prepare_select(const pbsa_config* cfg, const void* q, int q_frames, const void* k_local,
                       int local_frames, int ring_head, const int32_t* idx, int idx_stride,
                       const int32_t* cnt, const float* scores, Geo* geo, int* k,
                       size_t* scratch_bytes, size_t* key_offset) {
    int rc = validate(cfg);
    if (rc != PBSA_OK) return rc;
    const Geo g = make_geo(cfg);
    if ((rc = check_window(cfg, g, q_frames, local_frames, ring_head)) != PBSA_OK) return rc;
    REQUIRE_PTR(q);
    REQUIRE_PTR(k_local);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(cnt);
    OPTIONAL_PTR(scores);
    const int kk = topk_count(cfg, local_frames);
    if (idx_stride < kk) return fail(PBSA_ERR_ARG, "idx_stride %d < k %d", idx_stride, kk);
    const int nl = local_frames / g.bt * g.nbf;
    if (score_topk_smem_bytes(g, nl) > 227 * 1024)
        return fail(PBSA_ERR_UNSUPPORTED, "%d local blocks do not fit the scoring kernel", nl);
    *geo = g;
    *k = kk;
    *scratch_bytes = select_ws(g, q_frames);
    *key_offset = align256(sizeof(float) * (size_t)g.B * g.H * (q_frames / g.bt) * g.nbf * g.D);
    return PBSA_OK;
}

}  // namespace pbsa
