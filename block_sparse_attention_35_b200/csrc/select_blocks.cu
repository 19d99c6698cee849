// select_blocks.cu - PBSA block selection on sm_100a.
//
// Sparse Forcing (pith.science abstract): inside each sliding local window the
// computation is restricted to a dynamically selected neighbourhood; the project page
// calls it learned top-k selection with local_block_sparse_topk_ratio.  Block score =
// mean-pooled query block . mean-pooled key block / sqrt(D); the k best blocks (score
// descending, lower id first on ties) are kept.
//
// Two kernels:
//  1. pool_kernel: one CTA per (block, batch); each thread owns 8 consecutive channels of
//     the token's [H, D] row and streams the block's valid tokens (all bt frames of its
//     frame group) with 16-byte loads, so a CTA reads whole 3 KB token rows (all heads) -
//     fully coalesced, one HBM pass over Q and the window's K.  Means go to fp32
//     workspace; key means are stored by physical ring frame group, so a caller can keep
//     them across chunks and pool only the frames it appends (pbsa_pool_keys +
//     pbsa_select_blocks_pooled).
//  2. score_topk_kernel: one CTA per (8 query blocks, head, batch); the head's pooled keys
//     sit in shared memory (rows padded to D+1 floats: conflict-free), one warp per query
//     block computes its N_L scores, ranks every candidate by counting the candidates that
//     beat it (exact, deterministic, no sort), and writes the winners in ascending id
//     order with ballots.
#include <cuda_bf16.h>

#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

struct PoolParams {
    Geo g;
    const __nv_bfloat16* q;
    const __nv_bfloat16* kl;
    int q_frames;           // query frames to pool (0: none)
    int k_first, k_frames;  // ring frames k_first, k_first+1, ... (mod W) of K to pool
    float* qbar;  // [B, H, QB, D]
    float* kbar;  // [B, H, Wg*NB, D], by physical ring frame group
};

// ROWS rows in flight per thread: 16 when the CTA has at most 512 threads (H*D <= 4096),
// else 8 so that 1024 threads fit in the register file.
template <int ROWS>
__global__ void __launch_bounds__(ROWS > 8 ? 512 : 1024) pool_kernel(PoolParams p) {
    const Geo& g = p.g;
    const int qb_total = p.q_frames / g.bt * g.nbf;
    const int blk = blockIdx.x;
    const int b = blockIdx.y;
    const int hd = g.H * g.D;
    const int t = threadIdx.x;
    if (t * 8 >= hd) return;

    const __nv_bfloat16* src;
    long long frame;  // first frame of the block's group inside the source tensor
    int i_in_frame;
    float* dst;
    int local_id, n_of_kind;
    if (blk < qb_total) {
        frame = (long long)b * p.q_frames + (long long)(blk / g.nbf) * g.bt;
        i_in_frame = blk % g.nbf;
        src = p.q;
        dst = p.qbar;
        local_id = blk;
        n_of_kind = qb_total;
    } else {
        const int j = blk - qb_total;  // j-th block of the K frame groups being pooled
        const int phys = (p.k_first / g.bt + j / g.nbf) % g.Wg;
        frame = (long long)b * g.W + (long long)phys * g.bt;
        i_in_frame = j % g.nbf;
        src = p.kl;
        dst = p.kbar;
        local_id = phys * g.nbf + i_in_frame;
        n_of_kind = g.Wg * g.nbf;
    }
    const BlockBox bb = block_box(g, i_in_frame);
    const int y0 = bb.y0, x0 = bb.x0, hv = bb.hv, wv = bb.wv;
    const int plane = hv * wv;
    const int n = g.bt * plane;

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    const __nv_bfloat16* base = src + frame * g.tf * (long long)hd + t * 8;
    // rows are summed in order, as append_kernel does
    for (int r0 = 0; r0 < n; r0 += ROWS) {
        uint4 v[ROWS];
#pragma unroll
        for (int u = 0; u < ROWS; ++u) {
            const int r = r0 + u;
            if (r < n) {
                const int t = r / plane, y = y0 + (r % plane) / wv, x = x0 + r % wv;
                v[u] = __ldg(reinterpret_cast<const uint4*>(base + ((long long)t * g.tf + y * g.fw + x) * hd));
            }
        }
#pragma unroll
        for (int u = 0; u < ROWS; ++u) {
            if (r0 + u < n) {
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h2[e]);
                    acc[2 * e] += f.x;
                    acc[2 * e + 1] += f.y;
                }
            }
        }
    }
    const int h = (t * 8) / g.D, d0 = (t * 8) % g.D;
    float* out = dst + (((long long)b * g.H + h) * n_of_kind + local_id) * g.D + d0;
    const float c = static_cast<float>(n);
    float4 o0 = make_float4(acc[0] / c, acc[1] / c, acc[2] / c, acc[3] / c);
    float4 o1 = make_float4(acc[4] / c, acc[5] / c, acc[6] / c, acc[7] / c);
    reinterpret_cast<float4*>(out)[0] = o0;
    reinterpret_cast<float4*>(out)[1] = o1;
}

constexpr int kQbPerCta = 8;   // query blocks (= warps) per CTA
constexpr int kMaxChunks = 16; // candidates per warp lane: N_L <= 512

struct ScoreParams {
    Geo g;
    const float* qbar;
    const float* kbar;  // [B, H, Wg*NB, D] by physical ring frame group
    int ring_head;
    int qb_total, nl, k;
    int32_t* idx;
    int idx_stride;
    int32_t* cnt;
    float* scores;
};

__global__ void __launch_bounds__(256) score_topk_kernel(ScoreParams p) {
    extern __shared__ float sm[];
    const Geo& g = p.g;
    const int D = g.D;
    const int b = blockIdx.z, h = blockIdx.y;
    const int bh = b * g.H + h;
    const int nl = p.nl;
    float* kb = sm;                               // [nl][D+1]
    float* qs = kb + (((size_t)nl * (D + 1) + 3) & ~(size_t)3);  // [8][D], 16-byte aligned
    float* sc = qs + kQbPerCta * D;               // [8][nl]

    // 16-byte loads, several in flight per thread (the copy is latency-bound otherwise);
    // rows are stored padded to D + 1 floats so that the dot products below are conflict-free
    // logical window block j (oldest frame group first) is ring row
    // ((ring_head / bt + j / NB) % Wg, j % NB)
    const float* kbh = p.kbar + (size_t)bh * g.Wg * g.nbf * D;
    const int n4 = nl * D / 4;
    const int head_g = p.ring_head / g.bt;
#pragma unroll 4
    for (int e = threadIdx.x; e < n4; e += blockDim.x) {
        const int j = (4 * e) / D, d = (4 * e) % D;
        const int row = ((head_g + j / g.nbf) % g.Wg) * g.nbf + j % g.nbf;
        const float4 v = __ldg(reinterpret_cast<const float4*>(kbh + (size_t)row * D + d));
        float* dst = kb + j * (D + 1) + d;
        dst[0] = v.x;
        dst[1] = v.y;
        dst[2] = v.z;
        dst[3] = v.w;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = blockIdx.x * kQbPerCta + warp;
    if (qb < p.qb_total) {
        const float* qsrc = p.qbar + ((size_t)bh * p.qb_total + qb) * D;
        for (int d = lane; d < D; d += 32) qs[warp * D + d] = qsrc[d];
    }
    __syncthreads();
    if (qb >= p.qb_total) return;

    const float* qrow = qs + warp * D;
    float* srow = sc + warp * nl;
    const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
    for (int j = lane; j < nl; j += 32) {
        const float* kr = kb + j * (D + 1);
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; d += 4) {
            const float4 q4 = *reinterpret_cast<const float4*>(qrow + d);
            acc0 = fmaf(q4.x, kr[d], acc0);
            acc1 = fmaf(q4.y, kr[d + 1], acc1);
            acc0 = fmaf(q4.z, kr[d + 2], acc0);
            acc1 = fmaf(q4.w, kr[d + 3], acc1);
        }
        srow[j] = (acc0 + acc1) * inv_sqrt_d;
    }
    __syncwarp();

    // rank of candidate j = number of candidates that come before it
    int selected_bits = 0;  // bit c: candidate 32c + lane is selected
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
        const int j = c * 32 + lane;
        if (c * 32 < nl && j < nl) {
            const float sj = srow[j];
            int rank = 0;
            for (int i = 0; i < nl; ++i) {
                const float si = srow[i];
                rank += (si > sj) || (si == sj && i < j);
            }
            if (rank < p.k) selected_bits |= 1 << c;
        }
    }
    int32_t* out = p.idx + ((size_t)bh * p.qb_total + qb) * p.idx_stride;
    int base = 0;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
        if (c * 32 < nl) {
            const bool sel = (selected_bits >> c) & 1;
            const unsigned m = __ballot_sync(0xffffffffu, sel);
            if (sel) out[base + __popc(m & ((1u << lane) - 1u))] = c * 32 + lane;
            base += __popc(m);
        }
    }
    if (lane == 0) p.cnt[(size_t)bh * p.qb_total + qb] = p.k;
    if (p.scores) {
        float* so = p.scores + ((size_t)bh * p.qb_total + qb) * nl;
        for (int j = lane; j < nl; j += 32) so[j] = srow[j];
    }
}

// Every window block selected (k = N_L, no scores asked for): the list is 0..N_L-1.
__global__ void __launch_bounds__(256) select_all_kernel(int32_t* __restrict__ idx, int idx_stride,
                                                         int32_t* __restrict__ cnt, long long rows, int nl) {
    const long long r = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    for (int j = lane; j < nl; j += 32) idx[r * idx_stride + j] = j;
    if (lane == 0) cnt[r] = nl;
}

}  // namespace

cudaError_t launch_select_all(const Geo& g, int qb, int nl, int32_t* idx, int idx_stride, int32_t* cnt,
                              cudaStream_t st) {
    const long long rows = (long long)g.B * g.H * qb;   // one warp per (b, h, query block)
    select_all_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(idx, idx_stride, cnt, rows, nl);
    return cudaGetLastError();
}

cudaError_t launch_pool(const Geo& g, const __nv_bfloat16* q, int q_frames,
                        const __nv_bfloat16* k_local, int k_first, int k_frames,
                        float* qbar, float* kbar, cudaStream_t st) {
    PoolParams p{g, q, k_local, q_frames, k_first, k_frames, qbar, kbar};
    const int nblk = (q_frames + k_frames) / g.bt * g.nbf;
    if (nblk == 0) return cudaSuccess;
    const int threads = (g.H * g.D / 8 + 31) / 32 * 32;
    if (threads <= 512)
        pool_kernel<16><<<dim3(nblk, g.B), threads, 0, st>>>(p);
    else
        pool_kernel<8><<<dim3(nblk, g.B), threads, 0, st>>>(p);
    return cudaGetLastError();
}

size_t score_topk_smem_bytes(const Geo& g, int nl) {
    return sizeof(float) * ((((size_t)nl * (g.D + 1) + 3) & ~(size_t)3) + (size_t)kQbPerCta * g.D +
                            (size_t)kQbPerCta * nl);
}

cudaError_t launch_score_topk(const Geo& g, const float* qbar, const float* kbar, int ring_head, int qb,
                              int nl, int k, int32_t* idx, int idx_stride, int32_t* cnt, float* scores,
                              cudaStream_t st) {
    ScoreParams p{g, qbar, kbar, ring_head, qb, nl, k, idx, idx_stride, cnt, scores};
    const size_t smem = score_topk_smem_bytes(g, nl);
    cudaError_t e = cudaFuncSetAttribute(score_topk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((qb + kQbPerCta - 1) / kQbPerCta, g.H, g.B);
    score_topk_kernel<<<grid, 32 * kQbPerCta, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace pbsa
