// cache_update.cu - PBSA window slide and persistent-cache merge on sm_100a.
//
// Sparse Forcing (pith.science abstract): the persistent blocks are compressed, preserved
// and updated; the algorithm fragment on the same page updates P and L in the t=0 pass.
// When the oldest frames leave the local window, their blocks compete with the occupied
// persistent slots on accumulated attention mass; the best min(S, #candidates) stay.  The
// sink slots at the front of the store (project page: the "sink" sparsity pattern) take
// no part: they are never candidates and never free.
//
// Two kernels:
//  1. merge_rank_kernel, one CTA per (head, batch): candidates (occupied slots in slot
//     order, then the evicted blocks in logical id order) are ranked by counting the
//     candidates that beat each one (score descending, earlier candidate first on ties);
//     one warp then builds the free-slot list (empty slots ascending, then dropped slots
//     ascending) and the admission list with ballots, and the metadata is rewritten.  The
//     evicted blocks' mass entries are cleared for the frames that will reuse the slots.
//  2. merge_copy_kernel, one CTA per (admission, head, batch): copies the admitted block's
//     valid tokens from the ring into its slot with 16-byte loads/stores (a warp moves two
//     256-byte token rows per instruction) and zero-fills the slot's tail rows.
#include <cuda_bf16.h>

#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

struct MergeParams {
    Geo g;
    int local_frames, ring_head, n_ev_frames, first_frame_global;
    float* mass_local;
    int32_t* pers_len;
    float* pers_score;
    int32_t* pers_src;
    int32_t* upd;
    int32_t* n_upd;
};

constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads) merge_rank_kernel(MergeParams p) {
    extern __shared__ uint8_t smraw[];
    const Geo& g = p.g;
    const int S = g.S;
    const int h = blockIdx.x, b = blockIdx.y, bh = b * g.H + h;
    const int n_ev = p.n_ev_frames / g.bt * g.nbf;
    const int head_g = p.ring_head / g.bt;
    const int ncand_max = S + n_ev;
    float* sc = reinterpret_cast<float*>(smraw);            // [S + n_ev] candidate scores
    int* cid = reinterpret_cast<int*>(sc + ncand_max);      // [S + n_ev] slot or block id
    int* kept = cid + ncand_max;                            // [S + n_ev]
    int* len = kept + ncand_max;                            // [S]
    int* freel = len + S;                                   // [S]
    __shared__ int s_nocc, s_nempty;

    for (int s = threadIdx.x; s < S; s += blockDim.x) len[s] = p.pers_len[(size_t)bh * S + s];
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        // occupied slots -> candidates 0..n_occ-1; empty slots -> head of the free list
        // (the sink slots 0 .. n_sink-1 are neither)
        int occ = 0, emp = 0;
        for (int s0 = g.n_sink; s0 < S; s0 += 32) {
            const int s = s0 + lane;
            const bool valid = s < S;
            const bool o = valid && len[s] > 0;
            const bool e = valid && len[s] <= 0;
            const unsigned mo = __ballot_sync(0xffffffffu, o);
            const unsigned me = __ballot_sync(0xffffffffu, e);
            const unsigned lt = (1u << lane) - 1u;
            if (o) {
                const int c = occ + __popc(mo & lt);
                cid[c] = s;
                sc[c] = p.pers_score[(size_t)bh * S + s];
            }
            if (e) freel[emp + __popc(me & lt)] = s;
            occ += __popc(mo);
            emp += __popc(me);
        }
        if (lane == 0) {
            s_nocc = occ;
            s_nempty = emp;
        }
    }
    __syncthreads();
    const int n_occ = s_nocc;
    const int ncand = n_occ + n_ev;
    for (int j = threadIdx.x; j < n_ev; j += blockDim.x) {
        const int phys = (head_g + j / g.nbf) % g.Wg;
        const size_t mi = ((size_t)bh * g.Wg + phys) * g.nbf + j % g.nbf;
        cid[n_occ + j] = j;
        sc[n_occ + j] = p.mass_local[mi];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < ncand; c += blockDim.x) {
        const float s = sc[c];
        int rank = 0;
        for (int o = 0; o < ncand; ++o) rank += (sc[o] > s) || (sc[o] == s && o < c);
        kept[c] = rank < S - g.n_sink;
    }
    __syncthreads();
    if (warp == 0) {
        // free list: empties (already at the head), then dropped slots ascending
        int nfree = s_nempty;
        for (int c0 = 0; c0 < n_occ; c0 += 32) {
            const int c = c0 + lane;
            const bool dropped = c < n_occ && !kept[c];
            const unsigned m = __ballot_sync(0xffffffffu, dropped);
            if (dropped) {
                const int s = cid[c];
                freel[nfree + __popc(m & ((1u << lane) - 1u))] = s;
                p.pers_len[(size_t)bh * S + s] = 0;
                p.pers_score[(size_t)bh * S + s] = 0.f;
                p.pers_src[(size_t)bh * S + s] = -1;
            }
            nfree += __popc(m);
        }
        __syncwarp();
        // admissions: kept evicted blocks in id order take the free slots in order
        int nadm = 0;
        for (int c0 = n_occ; c0 < ncand; c0 += 32) {
            const int c = c0 + lane;
            const bool adm = c < ncand && kept[c];
            const unsigned m = __ballot_sync(0xffffffffu, adm);
            if (adm) {
                const int k = nadm + __popc(m & ((1u << lane) - 1u));
                const int j = cid[c];
                const int s = freel[k];
                const int i = j % g.nbf;
                const BlockBox bb = block_box(g, i);
                p.pers_len[(size_t)bh * S + s] = g.bt * bb.hv * bb.wv;
                p.pers_score[(size_t)bh * S + s] = sc[c];
                p.pers_src[(size_t)bh * S + s] = (p.first_frame_global / g.bt + j / g.nbf) * g.nbf + i;
                p.upd[((size_t)bh * n_ev + k) * 2 + 0] = s;
                p.upd[((size_t)bh * n_ev + k) * 2 + 1] = j;
            }
            nadm += __popc(m);
        }
        if (lane == 0) p.n_upd[bh] = nadm;
    }
    __syncthreads();
    // the evicted frames' slots of the ring start over for the next frames
    for (int j = threadIdx.x; j < n_ev; j += blockDim.x) {
        const int phys = (head_g + j / g.nbf) % g.Wg;
        p.mass_local[((size_t)bh * g.Wg + phys) * g.nbf + j % g.nbf] = 0.f;
    }
}

struct CopyParams {
    Geo g;
    int ring_head, n_ev;
    const __nv_bfloat16* kl;
    const __nv_bfloat16* vl;
    __nv_bfloat16* kp;
    __nv_bfloat16* vp;
    const int32_t* upd;
    const int32_t* n_upd;
};

__global__ void __launch_bounds__(256) merge_copy_kernel(CopyParams p) {
    const Geo& g = p.g;
    const int k = blockIdx.x, h = blockIdx.y, b = blockIdx.z, bh = b * g.H + h;
    if (k >= p.n_upd[bh]) return;
    const int slot = p.upd[((size_t)bh * p.n_ev + k) * 2 + 0];
    const int j = p.upd[((size_t)bh * p.n_ev + k) * 2 + 1];
    // first ring frame of the block's frame group (groups never wrap: W and ring_head are
    // multiples of bt)
    const int phys = (p.ring_head + (j / g.nbf) * g.bt) % g.W;
    const BlockBox bb = block_box(g, j % g.nbf);
    const int y0 = bb.y0, x0 = bb.x0, wv = bb.wv, plane = bb.hv * bb.wv, c = g.bt * plane;
    const int cpr = g.D / 8;  // 16-byte chunks per token row
    const size_t frame_base = ((size_t)b * g.W + phys) * g.tf;
    const size_t slot_base = ((size_t)bh * g.S + slot) * 64;
    for (int e = threadIdx.x; e < 64 * cpr; e += blockDim.x) {
        const int row = e / cpr, ch = e % cpr;
        uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
        if (row < c) {
            const int t = row / plane, y = y0 + (row % plane) / wv, x = x0 + row % wv;
            const size_t src = ((frame_base + (size_t)t * g.tf + (size_t)y * g.fw + x) * g.H + h) * g.D + ch * 8;
            kv = __ldg(reinterpret_cast<const uint4*>(p.kl + src));
            vv = __ldg(reinterpret_cast<const uint4*>(p.vl + src));
        }
        const size_t dst = (slot_base + row) * g.D + ch * 8;
        *reinterpret_cast<uint4*>(p.kp + dst) = kv;
        *reinterpret_cast<uint4*>(p.vp + dst) = vv;
    }
}

}  // namespace

cudaError_t launch_cache_update(const Geo& g, const __nv_bfloat16* k_local,
                                const __nv_bfloat16* v_local, int local_frames, int ring_head,
                                float* mass_local, int n_evict_frames, int first_frame_global,
                                __nv_bfloat16* k_pers, __nv_bfloat16* v_pers, int32_t* pers_len,
                                float* pers_score, int32_t* pers_src, int32_t* upd,
                                int32_t* n_upd, cudaStream_t st) {
    const int n_ev = n_evict_frames / g.bt * g.nbf;
    if (n_ev == 0) return cudaSuccess;
    MergeParams mp{g, local_frames, ring_head, n_evict_frames, first_frame_global,
                   mass_local, pers_len, pers_score, pers_src, upd, n_upd};
    const size_t smem = (size_t)(g.S + n_ev) * 12 + (size_t)g.S * 8;
    cudaError_t e = cudaFuncSetAttribute(merge_rank_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    merge_rank_kernel<<<dim3(g.H, g.B), kMergeThreads, smem, st>>>(mp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CopyParams cp{g, ring_head, n_ev, k_local, v_local, k_pers, v_pers, upd, n_upd};
    merge_copy_kernel<<<dim3(n_ev, g.H, g.B), 256, 0, st>>>(cp);
    return cudaGetLastError();
}

}  // namespace pbsa
