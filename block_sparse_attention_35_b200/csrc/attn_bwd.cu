// attn_bwd.cu - PBSA backward on sm_100a (TMA + tcgen05 + TMEM).
//
// Sparse Forcing project page (kernel features): full gradient support for training.
// Gradients of sum(O * dO) with the block selection held fixed:
//   P  = exp(S - lse) with S = Q K^T / sqrt(D)   (recomputed from the forward's lse)
//   dV = P^T dO,   dP = dO V^T,   Delta = rowsum(dO * O),   dS = P * (dP - Delta)
//   dQ = dS K / sqrt(D),   dK = dS^T Q / sqrt(D)
// Two launches:
//  1. delta_kernel: Delta per query row (one pass over O and dO); it also zeroes dQ.
//  2. bwd_kernel: one CTA per key tile (128 keys: 16 compacted 8-row groups of the
//     persistent slots, or a pair of local blocks).  K and V stay in shared memory while
//     the CTA walks the 64-row query blocks that attend to its keys (every query block for
//     persistent keys; for local blocks the query blocks that selected either block).  Per
//     query block u:
//       S^T = K Q_u^T, dP^T = V dO_u^T     128 keys x 64 queries, into one of two TMEM buffers
//       8 element warps                    P^T and dS^T (bf16, packed over S^T in TMEM; dS^T
//                                          also into a 128B-swizzled shared-memory tile)
//       dV += P^T dO_u, dK += dS^T Q_u     (A from TMEM)
//       dQ^T_u = K^T dS^T                  (both from shared memory, into the buffer's dP^T
//                                          columns)
//       4 dQ warps                         read dQ^T_u, stage it as the query block's box and
//                                          add it into dQ with TMA reductions (a query row's
//                                          other key tiles add theirs, so dQ is summed in no
//                                          fixed order)
//     Every tensor-core product is computed once: five GEMMs per (key tile, query block).
//     S^T of block u + 2 is computed while the element warps work on block u + 1, and its
//     dP^T as soon as the dQ warps have read dQ^T of block u out of the same columns.
// Warp roles: 0-7 element warps, 8 TMA producer, 9 MMA, 10-13 dQ warps (one per TMEM
// lane quarter).  Persistent slots of any length 1..64 are streamed as ceil(len / 8) groups;
// key rows of a partial last group past the slot's length are masked (P and dS exactly zero),
// so they only need to hold finite values.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

constexpr uint32_t kHalf = 128 * 128;   // 128 rows x 64 bf16 channels
// Warp roles: 8 element warps (two per TMEM lane quarter, each over 32 query columns),
// one TMA producer warp, one MMA warp, four dQ warps.
constexpr int kElemWarps = 8;
constexpr int kColsW = 256 / kElemWarps;  // query columns per element warp (64 per block)
static_assert(kColsW % 16 == 0 && kColsW * (kElemWarps / 4) == 64, "element warp columns");

// tcgen05.ld of N (16 or 32) consecutive columns of the warp's lane quarter
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 32, "16 or 32 columns");
    if constexpr (N == 32)
        tmem_ld32(taddr, r);
    else
        tmem_ld16(taddr, r);
}
constexpr int kProdWarp = kElemWarps;
constexpr int kMmaWarp = kElemWarps + 1;
constexpr int kDqWarp0 = kElemWarps + 2;
constexpr int kDqWarps = 4;
constexpr int kThreads = 32 * (kElemWarps + 2 + kDqWarps);
constexpr float kLog2e = 1.4426950408889634f;


// ----------------------------------------------------------------------- delta
// Delta per (token, head) row and dQ := 0 for the same row (the key-tile CTAs add into it).
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                    const __nv_bfloat16* __restrict__ d_o,
                                                    float* __restrict__ delta, float* __restrict__ dq,
                                                    int nq, int H, int D, long long nrows) {
    // one row (token, head) per 16 threads, 8 channels per thread per step
    const long long row = (long long)blockIdx.x * 16 + threadIdx.x / 16;
    const int sub = threadIdx.x % 16;
    float acc = 0.f;
    if (row < nrows) {
        const __nv_bfloat16* a = o + row * D;
        const __nv_bfloat16* b = d_o + row * D;
        float* z = dq + row * D;
        for (int c = sub * 8; c < D; c += 128) {
            const uint4 va = __ldg(reinterpret_cast<const uint4*>(a + c));
            const uint4 vb = __ldg(reinterpret_cast<const uint4*>(b + c));
            reinterpret_cast<float4*>(z + c)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4*>(z + c)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&va);
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&vb);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fa = __bfloat1622float2(pa[e]);
                const float2 fb = __bfloat1622float2(pb[e]);
                acc = fmaf(fa.x, fb.x, acc);
                acc = fmaf(fa.y, fb.y, acc);
            }
        }
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, 16);
    if (row < nrows && sub == 0) {
        // row = (b * nq + t) * H + h  ->  delta[(b * H + h) * nq + t]
        const long long bt = row / H;
        const int h = (int)(row % H);
        const long long b = bt / nq, t = bt % nq;
        delta[(b * H + h) * nq + t] = acc;
    }
}

// --------------------------------------------------------- persistent group table
// Builds, with one warp, the compacted list of the occupied slots' 8-row groups
// (ceil(len / 8) per slot): the first row of each group in the [B*H*S*64, D] slot store,
// with the group's valid-row count & 7 in the low 3 bits (0 = all 8 rows valid; only a
// slot's last group can be partial).  Returns the group count.
__device__ int build_groups(const int32_t* pers_len, int bh, int S, int32_t* grp_row,
                            int32_t* status) {
    const int lane = threadIdx.x & 31;
    int run = 0;
    for (int s0 = 0; s0 < S; s0 += 32) {
        const int s = s0 + lane;
        int len = (s < S) ? pers_len[(size_t)bh * S + s] : 0;
        if (len < 0 || len > 64) {
            set_status(status, PBSA_ERR_DEVICE_CHECK);
            len = 0;
        }
        const int ng = (len + 7) >> 3;
        int inc = ng;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        const int gstart = run + inc - ng;
        for (int i = 0; i < ng; ++i)
            grp_row[gstart + i] = (((bh * S) + s) * 64 + 8 * i) | (min(8, len - 8 * i) & 7);
        run += __shfl_sync(0xffffffffu, inc, 31);
    }
    return run;
}

// Valid rows (1..8) of a group-table entry.
__device__ __forceinline__ int group_rows(int32_t entry) {
    const int nv = entry & 7;
    return nv ? nv : 8;
}

// Zeroes a CTA's operand tiles (bytes, a multiple of 16) with every thread, then orders
// those writes before the TMA copies and MMAs that follow.  Blocks of fewer than 64 tokens
// leave box rows that TMA never writes; they must hold finite values because masked
// columns multiply them by exact zeros.
__device__ __forceinline__ void zero_tiles(uint8_t* base, uint32_t bytes) {
    uint4* z = reinterpret_cast<uint4*>(base);
    for (uint32_t e = threadIdx.x; e < bytes / 16; e += blockDim.x) z[e] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
}

// ================================================================== key-tile CTA
// Query blocks arrive in kQst stages: Q and dO of a 64-row block are one TMA box each per
// 64 channels (16 KB for both halves of D), with the block's lse, Delta and row tokens.
constexpr int kQst = 3;
constexpr uint32_t kQBlk = 64 * 128;    // bytes of one query block, one 64-channel half
constexpr uint32_t kDsBuf = 128 * 128;  // dS^T of one query block: 128 keys x 64 queries bf16
constexpr int B_COUNT = 20;             // mbarrier slots reserved per CTA

struct BwdPlan {
    uint32_t k, v, q, dq_o, ds, lse, dl, grp_row, sub, bars, misc, dqs, total;
};

__host__ __device__ inline BwdPlan bwd_plan(int D, int S, int qb_total) {
    BwdPlan p;
    const uint32_t nh = D / 64;
    p.k = 0;
    p.v = p.k + nh * kHalf;
    p.q = p.v + nh * kHalf;                 // kQst stages of one query block's Q
    p.dq_o = p.q + kQst * nh * kQBlk;       // kQst stages of its dO
    p.ds = p.dq_o + kQst * nh * kQBlk;      // the dS^T tile (1024-byte aligned)
    p.lse = p.ds + kDsBuf;              // kQst x 64 fp32 (log2 units, +inf = padding)
    p.dl = p.lse + kQst * 64 * 4;           // kQst x 64 fp32 Delta
    p.grp_row = p.dl + kQst * 64 * 4;       // 8*S
    p.sub = p.grp_row + 4u * 8u * S;        // query blocks that see the keys: qb << 2 | bits
    p.bars = (p.sub + 4u * qb_total + 7u) & ~7u;
    p.misc = p.bars + 8u * B_COUNT;
    p.dqs = (p.misc + 4u * 8u + 1023u) & ~1023u;  // dQ staging: per 64 channels, 64 rows x 64 fp32
    p.total = p.dqs + 64u * 4u * D;
    return p;
}

struct BwdKernelArgs {
    BwdArgs a;
    int n_pt_max;  // persistent key tiles per (b, h)
    int n_kd_x;    // key-tile CTAs per (b, h): persistent + local key tiles
};

// Gradients of key tile cta_x of head h, batch b.
template <int D>
__device__ __forceinline__ void key_tile_body(const BwdKernelArgs& ka, const int cta_x, const int h,
                                              const int b) {
    constexpr int NH = D / 64;
    constexpr uint32_t TILE = NH * kHalf;
    constexpr uint32_t QSTAGE = NH * kQBlk;
    // TMEM: two buffers (buffer x at 128 x) of S^T (+0) and dP^T (+64) for a 64-query block;
    // P^T is packed over S^T and dQ^T replaces dP^T; then the dV and dK accumulators
    constexpr uint32_t kTmDV = 256, kTmDK = 256 + D;
    const BwdArgs& a = ka.a;
    const Geo& g = a.g;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int S = g.S;
    const int qb_total = a.q_frames / g.bt * g.nbf;
    const BwdPlan PL = bwd_plan(D, S, qb_total);
    uint8_t* sK = sm + PL.k;
    uint8_t* sV = sm + PL.v;
    uint8_t* sQ = sm + PL.q;
    uint8_t* sDO = sm + PL.dq_o;
    uint8_t* sDS = sm + PL.ds;
    float* s_lse = reinterpret_cast<float*>(sm + PL.lse);
    float* s_dl = reinterpret_cast<float*>(sm + PL.dl);
    int32_t* grp_row = reinterpret_cast<int32_t*>(sm + PL.grp_row);
    int32_t* sub = reinterpret_cast<int32_t*>(sm + PL.sub);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL.bars);
    int* misc = reinterpret_cast<int*>(sm + PL.misc);
    volatile int* abort_flag = misc + 1;

    const int bh = b * g.H + h;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nq = a.q_frames * g.tf;
    const int nl = a.local_frames / g.bt * g.nbf;
    const uint32_t box_bytes = static_cast<uint32_t>(g.brows) * 128u;  // one block, one 64-channel half
    const bool pers_tile = cta_x < ka.n_pt_max;
    const int tile = pers_tile ? cta_x : cta_x - ka.n_pt_max;

    uint64_t* kv_full = &bars[0];      // K and V tiles of this CTA (once)
    uint64_t* qd_full = &bars[1];      // [kQst] Q + dO + lse/Delta of a query block
    uint64_t* qd_empty = &bars[4];     // [kQst] dV / dK of that block done
    uint64_t* sdp_full = &bars[7];     // [2] S^T and dP^T of a query block in TMEM buffer x
    uint64_t* pds_full = &bars[9];     // [2] P^T and dS^T written (one arrival per element warp)
    uint64_t* dq_full = &bars[11];     // [2] dQ^T of a query block computed (the dS^T tile free)
    uint64_t* dq_free = &bars[13];     // [2] dQ^T read out of TMEM (one arrival per dQ warp)
    uint64_t* pass_done = &bars[15];   // MMAs of the last query block done (one phase)
    uint64_t* drain = &bars[16];
    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kQst; ++s) {
            mbar_init(&qd_full[s], 1 + 32);  // producer expect_tx + 32 lse/Delta loaders
            mbar_init(&qd_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sdp_full[x], 1);
            mbar_init(&pds_full[x], kElemWarps);
            mbar_init(&dq_full[x], 1);
            mbar_init(&dq_free[x], kDqWarps);
        }
        mbar_init(pass_done, 1);
        mbar_init(drain, 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    if (g.brows < 64) zero_tiles(sm + PL.k, PL.ds - PL.k);
    if (warp == kMmaWarp) tmem_alloc(reinterpret_cast<uint32_t*>(misc + 0), 512);

    // key set of this CTA
    int G = 0, L0 = -1, L1 = -1;
    if (pers_tile) {
        if (warp == 0) {
            G = build_groups(a.pers_len, bh, S, grp_row, a.status);
            if (lane == 0) misc[2] = G;
        }
    } else {
        L0 = 2 * tile;
        L1 = (2 * tile + 1 < nl) ? 2 * tile + 1 : -1;
    }
    __syncthreads();
    if (pers_tile) G = misc[2];
    // the query blocks that see these keys, with bit kb set when the block selected key
    // block kb (persistent keys: every query block, both bits).  Persistent tiles start their
    // walk at a tile-dependent block, so that the tiles of one head do not all add into the
    // same dQ rows at the same time.
    if (warp < 4) {
        int count = 0;
        for (int q0 = 0; q0 < qb_total; q0 += 128) {
            const int qb = q0 + threadIdx.x;
            int bits = 0;
            if (qb < qb_total) {
                if (pers_tile) {
                    bits = 3;
                } else {
                    const int c = min(max(a.cnt[(size_t)bh * qb_total + qb], 0), a.idx_stride);
                    const int32_t* row = a.idx + ((size_t)bh * qb_total + qb) * a.idx_stride;
                    for (int i = 0; i < c; ++i) {
                        const int v = row[i];
                        if (v == L0) bits |= 1;
                        if (L1 >= 0 && v == L1) bits |= 2;
                    }
                }
            }
            // block-wide compaction of the blocks with bits != 0 (4 warps)
            const unsigned m = __ballot_sync(0xffffffffu, bits != 0);
            __shared__ int wcount[4];
            if (lane == 0) wcount[warp] = __popc(m);
            named_bar_sync(1, 128);
            int base = count;
            for (int w = 0; w < warp; ++w) base += wcount[w];
            if (bits) {
                int pos = base + __popc(m & ((1u << lane) - 1u));
                if (pers_tile) pos = (pos + qb_total - tile % qb_total) % qb_total;
                sub[pos] = (qb << 2) | bits;
            }
            count += wcount[0] + wcount[1] + wcount[2] + wcount[3];
            named_bar_sync(1, 128);
        }
        if (threadIdx.x == 0) misc[3] = count;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(misc[0]);
    const int n_sub = misc[3];
    const bool live = pers_tile ? (tile * 16 < G) : true;

    if (live && warp == kProdWarp) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            mbar_arrive_expect_tx(kv_full, pers_tile ? 2 * TILE : 2 * 2 * NH * box_bytes);
            if (pers_tile) {
                tma_load_groups16<NH>(sK, kHalf, &a.tm_kp, &a.tm_kp64, grp_row, tile * 16, G, kv_full);
                tma_load_groups16<NH>(sV, kHalf, &a.tm_vp, &a.tm_vp64, grp_row, tile * 16, G, kv_full);
            } else {
                for (int kb = 0; kb < 2; ++kb) {
                    const int L = (kb == 1 && L1 >= 0) ? L1 : L0;
                    const BlockBox kbb = block_box(g, L % g.nbf);
                    const int fr = b * g.W + (a.ring_head + (L / g.nbf) * g.bt) % g.W;
                    for (int hh = 0; hh < NH; ++hh) {
                        tma_load_5d(sK + hh * kHalf + kb * (kHalf / 2), &a.tm_kl, kv_full, hh * 64, h,
                                    kbb.x0, kbb.y0, fr);
                        tma_load_5d(sV + hh * kHalf + kb * (kHalf / 2), &a.tm_vl, kv_full, hh * 64, h,
                                    kbb.x0, kbb.y0, fr);
                    }
                }
            }
        }
        __syncwarp();
        // in-block coordinates of this lane's two rows of a query block (rows lane, lane + 32)
        int rt[2], ry[2], rx[2];
        bool rin[2];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const int rr = lane + 32 * v;
            rx[v] = rr % g.bw;
            ry[v] = (rr / g.bw) % g.bh;
            rt[v] = rr / (g.bw * g.bh);
            rin[v] = rr < g.brows;
        }
        int issued = 0;
        for (int u = 0; u < n_sub; ++u) {
            const int st = u % kQst;
            const int qb = sub[u] >> 2;
            // lse (log2 units) and Delta of the block's 64 rows, read from global memory before
            // waiting for the stage so that their latency overlaps the wait; +inf lse masks
            // rows outside the frame
            const BlockBox qbb = block_box(g, qb % g.nbf);
            const size_t base = (size_t)bh * nq + (size_t)(qb / g.nbf) * g.bt * g.tf + qbb.y0 * g.fw + qbb.x0;
            float l2v[2], dlv[2];
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                l2v[v] = CUDART_INF_F;
                dlv[v] = 0.f;
                if (rin[v] && ry[v] < qbb.hv && rx[v] < qbb.wv) {
                    const size_t t = base + (size_t)rt[v] * g.tf + ry[v] * g.fw + rx[v];
                    l2v[v] = a.lse[t] * kLog2e;
                    dlv[v] = a.delta[t];
                }
            }
            if (u >= kQst) {
                const bool w = __all_sync(0xffffffffu, mbar_wait(&qd_empty[st], ((u / kQst) - 1) & 1, abort_flag, a.status));
                if (!w) break;
            }
            // copies issued by one elected lane of the converged warp
            const int f0 = b * a.q_frames + (qb / g.nbf) * g.bt;
            if (elect_one()) mbar_arrive_expect_tx(&qd_full[st], 2 * NH * box_bytes);
            __syncwarp();
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                if (elect_one())
                    tma_load_5d(sQ + st * QSTAGE + hh * kQBlk, &a.tm_q, &qd_full[st], hh * 64, h, qbb.x0, qbb.y0, f0);
                __syncwarp();
                if (elect_one())
                    tma_load_5d(sDO + st * QSTAGE + hh * kQBlk, &a.tm_do, &qd_full[st], hh * 64, h, qbb.x0, qbb.y0, f0);
                __syncwarp();
            }
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                s_lse[st * 64 + lane + 32 * v] = l2v[v];
                s_dl[st * 64 + lane + 32 * v] = dlv[v];
            }
            mbar_arrive(&qd_full[st]);
            ++issued;
        }
        if (lane == 0 && *abort_flag) {
            mbar_wait_drain(kv_full, 0, 100000000ull);
            for (int u = max(0, issued - kQst); u < issued; ++u)
                mbar_wait_drain(&qd_full[u % kQst], (u / kQst) & 1, 100000000ull);
        }
    } else if (live && warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA
        // the whole warp runs this (operands are warp-uniform); one elected lane issues each
        // MMA and commit
        {
            auto mma_ss = [&](uint32_t d, uint64_t a_, uint64_t b_, uint32_t id, uint32_t acc) {
                if (elect_one()) umma_ss(d, a_, b_, id, acc);
                __syncwarp();
            };
            auto mma_ts = [&](uint32_t d, uint32_t a_, uint64_t b_, uint32_t id, uint32_t acc) {
                if (elect_one()) umma_ts(d, a_, b_, id, acc);
                __syncwarp();
            };
            auto commit = [&](uint64_t* bar) {
                if (elect_one()) umma_commit(bar);
                __syncwarp();
            };
            auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.status));
            };
            constexpr uint32_t id_s = idesc_bf16(128, 64, false, false);   // 128 keys x 64 queries
            constexpr uint32_t id_g = idesc_bf16(128, D, false, true);      // dV, dK: B = dO / Q MN-major
            constexpr uint32_t id_q = idesc_bf16(128, 64, true, true);      // dQ^T: A = K^T, B = dS^T MN-major
            bool ok = wwait(kv_full, 0);
            const uint32_t kb = smem_u32(sK), vb = smem_u32(sV);
            // S^T = K Q_u^T into TMEM buffer u & 1 (columns +0), dP^T = V dO_u^T (+64)
            auto issue_s = [&](int u) -> bool {
                const int st = u % kQst;
                if (!wwait(&qd_full[st], (u / kQst) & 1)) return false;
                tc_fence_after();
                const uint32_t qs = smem_u32(sQ + st * QSTAGE);
                const uint32_t buf = tmem + 128 * (u & 1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ka_ = (kk >> 2) * kHalf + (kk & 3) * 32;   // K tile: 128 rows
                    const uint32_t kq = (kk >> 2) * kQBlk + (kk & 3) * 32;    // Q block: 64 rows
                    mma_ss(buf, sdesc_make(sdesc_lo(kb, 16) + (ka_ >> 4)), sdesc_make(sdesc_lo(qs, 16) + (kq >> 4)),
                            id_s, kk > 0);
                }
                return true;
            };
            auto issue_dp = [&](int u) {
                const int st = u % kQst;
                const uint32_t os = smem_u32(sDO + st * QSTAGE);
                const uint32_t buf = tmem + 128 * (u & 1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ka_ = (kk >> 2) * kHalf + (kk & 3) * 32;
                    const uint32_t kq = (kk >> 2) * kQBlk + (kk & 3) * 32;
                    mma_ss(buf + 64, sdesc_make(sdesc_lo(vb, 16) + (ka_ >> 4)), sdesc_make(sdesc_lo(os, 16) + (kq >> 4)),
                            id_s, kk > 0);
                }
                commit(&sdp_full[u & 1]);
            };
            for (int u = 0; ok && u < min(2, n_sub); ++u) {
                ok = issue_s(u);
                if (ok) issue_dp(u);
            }
            // Per query block u: dQ^T, dV and dK of u, then S^T of u + 2 into the same buffer
            // (it overwrites P^T(u) only after dV(u) has read it: the tensor pipe runs one
            // thread's MMAs in issue order), then, once the dQ warps have read dQ^T(u) out of
            // the dP^T columns, dP^T of u + 2.
            for (int u = 0; ok && u < n_sub; ++u) {
                const int st = u % kQst;
                if (!wwait(&pds_full[u & 1], (u >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t qs = smem_u32(sQ + st * QSTAGE), os = smem_u32(sDO + st * QSTAGE);
                const uint32_t ds = smem_u32(sDS);
                const uint32_t buf = tmem + 128 * (u & 1);
                // dQ^T = K^T dS^T: A = the K tile read MN-major (channels along M, the next 64
                // channels kHalf bytes on), B = dS^T read MN-major (queries along N); 16 keys
                // (2 KB of rows) per MMA
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(buf + 64, sdesc_make(sdesc_lo(kb, kHalf) + kk * 128),
                            sdesc_make(sdesc_lo(ds, kDsBuf) + kk * 128), id_q, kk > 0 ? 1u : 0u);
                // dQ^T first: its commit frees the dS^T tile for the next block's element warps
                commit(&dq_full[u & 1]);
                // B operands dO / Q read MN-major: 64 channels per 128-byte row, the next 64
                // channels kQBlk bytes on, 16 query rows per MMA
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tmem + kTmDV, buf + 16 * kk, sdesc_make(sdesc_lo(os, kQBlk) + kk * 128), id_g,
                            (u > 0 || kk > 0) ? 1u : 0u);
                // dK: A = dS^T, packed next to P^T in TMEM
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tmem + kTmDK, buf + 16 * kk + 8, sdesc_make(sdesc_lo(qs, kQBlk) + kk * 128), id_g,
                            (u > 0 || kk > 0) ? 1u : 0u);
                commit(&qd_empty[st]);
                // one phase, after the last block: the element warps may run two blocks ahead of
                // the dV/dK MMAs, so a per-block phase could not be waited on by parity alone
                if (u == n_sub - 1) commit(pass_done);
                if (u + 2 < n_sub) {
                    if (!issue_s(u + 2)) { ok = false; break; }
                    if (!wwait(&dq_free[u & 1], (u >> 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    issue_dp(u + 2);
                }
            }
            if (!ok) {
                commit(drain);
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else if (live && warp < kElemWarps) {
        // ------------------------------------------------------- element warps
        // warp w reads TMEM lanes 32 (w % 4).. (its key rows) and query columns
        // [kColsW (w / 4), +kColsW) of the block's S^T / dP^T; once it has read them it packs
        // P^T and dS^T (bf16) into its own S^T columns (per 16 queries: P^T into the first 8,
        // dS^T into the next 8; no other warp's input is overwritten) and writes dS^T into its
        // key rows of the block's dS^T tile in shared
        // memory: row r holds the 64 queries in 128 bytes, 16-byte chunk c stored at chunk
        // c ^ (r % 8) (128-byte swizzle)
        const int wq = warp & 3, cg = warp >> 2;
        const int r = 32 * wq + lane;
        const int c0 = kColsW * cg;         // first query column of this warp
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const float sl2 = kLog2e / sqrtf(static_cast<float>(D));
        bool key_valid;
        int kbr = 0;
        if (pers_tile) {
            const int gi = tile * 16 + (r >> 3);
            key_valid = gi < G && (r & 7) < group_rows(grp_row[gi]);
        } else {
            kbr = r >> 6;
            const int L = kbr ? L1 : L0;
            if (L < 0) {
                key_valid = false;
            } else {
                int tt, y, x;
                key_valid = block_row(g, block_box(g, L % g.nbf), r & 63, &tt, &y, &x);
            }
        }
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.status));
        };
        bool ok = true;
        for (int u = 0; u < n_sub; ++u) {
            const int st = u % kQst;
            // lse/Delta of this query block (written by the producer warp)
            if (!wwait(&qd_full[st], (u / kQst) & 1)) { ok = false; break; }
            if (!wwait(&sdp_full[u & 1], (u >> 1) & 1)) { ok = false; break; }
            // the dS^T tile is free once the dQ^T MMAs of block u - 1 are done
            if (u >= 1 && !wwait(&dq_full[(u - 1) & 1], ((u - 1) >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            const bool sel = key_valid && ((sub[u] >> kbr) & 1);
            // lse and Delta of the warp's 16 query columns: broadcast 16-byte loads (every lane
            // reads the same four columns)
            const float4* lse4 = reinterpret_cast<const float4*>(s_lse + st * 64 + c0);
            const float4* dl4 = reinterpret_cast<const float4*>(s_dl + st * 64 + c0);
            const uint32_t buf = 128 * (u & 1);
            uint32_t pk[kColsW / 2], dk[kColsW / 2];
            {
                uint32_t sv[kColsW], pv[kColsW];
                tmem_ld_cols(tmem + lane_base + buf + c0, sv);
                tmem_ld_cols(tmem + lane_base + buf + 64 + c0, pv);
                tmem_ld_wait();
#pragma unroll
                for (int e4 = 0; e4 < kColsW / 4; ++e4) {
                    const float4 l4 = lse4[e4], d4 = dl4[e4];
                    const float ls[4] = {l4.x, l4.y, l4.z, l4.w};
                    const float ds[4] = {d4.x, d4.y, d4.z, d4.w};
                    float p[4], d[4];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        // p is exactly 0 off the selection; dP^T there is finite (key rows past
                        // a slot's length are finite), so dS^T is exactly 0 as well
                        p[v] = sel ? fast_exp2(__uint_as_float(sv[4 * e4 + v]) * sl2 - ls[v]) : 0.f;
                        d[v] = p[v] * (__uint_as_float(pv[4 * e4 + v]) - ds[v]);
                    }
                    pk[2 * e4] = pack_bf16x2(p[0], p[1]);
                    pk[2 * e4 + 1] = pack_bf16x2(p[2], p[3]);
                    dk[2 * e4] = pack_bf16x2(d[0], d[1]);
                    dk[2 * e4 + 1] = pack_bf16x2(d[2], d[3]);
                }
            }
            // per 16 query columns: P^T packed into the first 8 of their S^T columns, dS^T
            // into the next 8 (the layout the dV and dK MMAs read)
#pragma unroll
            for (int j = 0; j < kColsW / 16; ++j) {
                uint32_t p8[8], d8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p8[e] = pk[8 * j + e];
                    d8[e] = dk[8 * j + e];
                }
                tmem_st8(tmem + lane_base + buf + c0 + 16 * j, p8);
                tmem_st8(tmem + lane_base + buf + c0 + 16 * j + 8, d8);
            }
            {
                uint8_t* row = sDS + r * 128;
#pragma unroll
                for (int j = 0; j < kColsW / 8; ++j)
                    *reinterpret_cast<uint4*>(row + ((((c0 >> 3) + j) ^ (r & 7)) << 4)) =
                        make_uint4(dk[4 * j], dk[4 * j + 1], dk[4 * j + 2], dk[4 * j + 3]);
            }
            fence_proxy_async_smem();
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pds_full[u & 1]);
        }
        ok = named_bar_and(2, 32 * kElemWarps, ok);
        if (ok && n_sub > 0) {
            ok = named_bar_and(2, 32 * kElemWarps, wwait(pass_done, 0));
            tc_fence_after();
        }
        if (ok) {
            // destination row of this key
            float* dk_row = nullptr;
            float* dv_row = nullptr;
            if (key_valid) {
                if (pers_tile) {
                    const size_t row = (size_t)(grp_row[tile * 16 + (r >> 3)] & ~7) + (r & 7);
                    dk_row = a.dk_pers + row * D;
                    dv_row = a.dv_pers + row * D;
                } else {
                    const int L = kbr ? L1 : L0;
                    const BlockBox kbb = block_box(g, L % g.nbf);
                    int tt, y, x;
                    block_row(g, kbb, r & 63, &tt, &y, &x);
                    // ring frame: the group's first frame (groups never wrap the ring) + tt
                    const int phys = (a.ring_head + (L / g.nbf) * g.bt) % g.W + tt;
                    const size_t tok = ((size_t)b * g.W + phys) * g.tf + (kbb.y0 + y) * g.fw + kbb.x0 + x;
                    dk_row = a.dk_local + (tok * g.H + h) * D;
                    dv_row = a.dv_local + (tok * g.H + h) * D;
                }
            }
            const float isd = 1.0f / sqrtf(static_cast<float>(D));
            // channel chunks of 16: chunk c goes to element warp column group c % (warps / 4)
            for (int c = cg; c < D / 16; c += kElemWarps / 4) {
                uint32_t v[16], w[16];
                if (n_sub > 0) {
                    tmem_ld16(tmem + lane_base + kTmDV + 16 * c, v);
                    tmem_ld16(tmem + lane_base + kTmDK + 16 * c, w);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = w[e] = 0u;
                }
                if (key_valid) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        *reinterpret_cast<float4*>(dv_row + 16 * c + e) =
                            make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                        __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                        *reinterpret_cast<float4*>(dk_row + 16 * c + e) =
                            make_float4(__uint_as_float(w[e]) * isd, __uint_as_float(w[e + 1]) * isd,
                                        __uint_as_float(w[e + 2]) * isd, __uint_as_float(w[e + 3]) * isd);
                    }
                }
            }
        }
    } else if (live && warp >= kDqWarp0) {
        // ---------------------------------------------------------------- dQ warps
        // warp w reads TMEM lanes 32 (w % 4).. = channels of dQ^T.  Per query block: read the
        // 64 query columns into registers and release them, write them into a staging tile
        // laid out as the query block's TMA box (per 64 channels: 64 rows of 64 fp32), and let
        // one thread add the tile into dQ with TMA reductions (one per 64 channels; rows
        // outside the frame are skipped).
        const int wq = warp & 3, dw = warp - kDqWarp0;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const int ch = 32 * wq + lane;
        const float isd = 1.0f / sqrtf(static_cast<float>(D));
        float* stage = reinterpret_cast<float*>(sm + PL.dqs);
        float* my_col = stage + (ch >> 6) * (64 * 64) + (ch & 63);   // column ch of row 0
        const bool issuer = dw == 0 && lane == 0;
        for (int u = 0; u < n_sub; ++u) {
            const bool okw = __all_sync(0xffffffffu, mbar_wait(&dq_full[u & 1], (u >> 1) & 1, abort_flag, a.status));
            // the four warps leave together if any wait gave up
            if (!named_bar_and(3, 32 * kDqWarps, okw)) break;
            tc_fence_after();
            const uint32_t col = tmem + lane_base + 128 * (u & 1) + 64;
            uint32_t v0[32], v1[32];
            tmem_ld32(col, v0);
            tmem_ld32(col + 32, v1);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dq_free[u & 1]);
            // the previous block's reductions have read the staging tile
            if (issuer) tma_store_wait_read();
            named_bar_sync(3, 32 * kDqWarps);
            if (ch < D) {
#pragma unroll
                for (int j = 0; j < 32; ++j) my_col[j * 64] = __uint_as_float(v0[j]) * isd;
#pragma unroll
                for (int j = 0; j < 32; ++j) my_col[(32 + j) * 64] = __uint_as_float(v1[j]) * isd;
            }
            fence_proxy_async_smem();
            named_bar_sync(3, 32 * kDqWarps);
            if (issuer) {
                const int qb = sub[u] >> 2;
                const BlockBox qbb = block_box(g, qb % g.nbf);
                const int f0 = b * a.q_frames + (qb / g.nbf) * g.bt;
                for (int hh = 0; hh < NH; ++hh)
                    tma_reduce_add_5d(&a.tm_dq, stage + hh * (64 * 64), hh * 64, h, qbb.x0, qbb.y0, f0);
                tma_store_commit();
            }
        }
        if (issuer) tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) bwd_kernel(const __grid_constant__ BwdKernelArgs ka) {
    const int r = blockIdx.x / ka.n_kd_x;
    key_tile_body<D>(ka, blockIdx.x % ka.n_kd_x, r % ka.a.g.H, r / ka.a.g.H);
}

template <class K, class A>
cudaError_t launch_k(K kernel, const A& args, dim3 grid, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, st>>>(args);
    return cudaGetLastError();
}

}  // namespace

size_t attn_bwd_smem_bytes(const Geo& g, int q_frames) {
    const size_t m = bwd_plan(g.D, g.S, q_frames / g.bt * g.nbf).total + 1024;
    return m < 120 * 1024 ? 120 * 1024 : m;
}

cudaError_t launch_attn_bwd(const BwdArgs& a, cudaStream_t st) {
    const Geo& g = a.g;
    const int nq = a.q_frames * g.tf;
    const long long nrows = (long long)g.B * nq * g.H;
    delta_kernel<<<(unsigned)((nrows + 15) / 16), 256, 0, st>>>(a.out, a.dout, a.delta, a.dq, nq, g.H, g.D, nrows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    BwdKernelArgs ka;
    ka.a = a;
    ka.n_pt_max = (g.S * 8 + 15) / 16;
    ka.n_kd_x = ka.n_pt_max + (a.local_frames / g.bt * g.nbf + 1) / 2;
    const size_t smem = attn_bwd_smem_bytes(g, a.q_frames);
    const long long ctas = (long long)ka.n_kd_x * g.H * g.B;
    if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    if (ctas == 0) return cudaSuccess;
    dim3 grid((unsigned)ctas);
    return g.D == 128 ? launch_k(bwd_kernel<128>, ka, grid, smem, st)
                      : launch_k(bwd_kernel<64>, ka, grid, smem, st);
}

}  // namespace pbsa
