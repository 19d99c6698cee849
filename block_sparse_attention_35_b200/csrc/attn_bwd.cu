// attn_bwd.cu - PBSA backward on sm_100a (TMA + tcgen05 + TMEM).
//
// Sparse Forcing project page (kernel features): full gradient support for training.
// Gradients of sum(O * dO) with the block selection held fixed:
//   P  = exp(S - lse) with S = Q K^T / sqrt(D)   (recomputed from the forward's lse)
//   dV = P^T dO,   dP = dO V^T,   Delta = rowsum(dO * O),   dS = P * (dP - Delta)
//   dQ = dS K / sqrt(D),   dK = dS^T Q / sqrt(D)
// Deterministic, no atomics, two launches: delta_kernel, then bwd_kernel, one grid whose
// first CTAs compute dQ and whose other CTAs compute dK/dV:
//  1. delta_kernel: Delta per query row (one pass over O and dO).
//  2. bwd_kernel, dK/dV CTAs (dkdv_body): one CTA per key tile (128 keys: 16 compacted
//     8-row groups of the persistent slots, or a pair of local blocks); it loops over the
//     64-row query blocks that attend to those keys (all of them for persistent keys; for
//     local blocks only the query blocks that selected either block).  S^T = K Q^T and
//     dP^T = V dO^T (128 keys x 64 queries) land in one of two TMEM buffers (lanes = keys);
//     16 element warps (a key-row quarter and 16 query columns each) form P^T and dS^T,
//     write them as bf16 back over S^T / dP^T, and two TS MMAs accumulate dV += P^T dO and
//     dK += dS^T Q in TMEM (dO and Q blocks read MN-major from shared memory).  The next
//     query block's S^T / dP^T are computed while the current one is in the element warps.
//  3. bwd_kernel, dQ CTAs (dq_body): one CTA per query tile (the forward's tiling); per key
//     tile S = Q K^T and dP = dO V^T in TMEM, the element warps (a query-row quarter and 32
//     key columns each) form dS, write it as bf16 over S, and a TS MMA accumulates
//     dQ += dS K (K read MN-major).  S is double-buffered in TMEM (S, S', dP, dQ = 512
//     columns) and the element warps release dP as soon as they have read it, so the next
//     key tile's S and dP are computed while the current tile's dS is formed.
// Warp roles in both parts: warps 0-15 elementwise (P, dS), warp 16 TMA producer, warp 17
// MMA.  The MMA thread issues the next tile's S / dP right after the current tile's
// gradient MMAs (the tensor pipe runs them in issue order), so only the element warps'
// work on a tile leaves the pipe idle.  Persistent slots of any length 1..64 are streamed
// as ceil(len / 8) groups; rows of a partial last group past the slot's length are masked
// (P and dS exactly zero), so they only need to hold finite values.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

constexpr uint32_t kHalf = 128 * 128;   // 128 rows x 64 bf16 channels
// Warp roles of the dK/dV and dQ kernels: 16 element warps (four per TMEM lane quarter, each
// over kCw columns), one TMA producer warp, one MMA warp.
constexpr int kNwq = 4;
constexpr int kElemWarps = 4 * kNwq;
constexpr int kCw = 128 / kNwq;
constexpr int kProdWarp = kElemWarps;
constexpr int kMmaWarp = kElemWarps + 1;
constexpr int kThreads = 32 * (kElemWarps + 2);
static_assert(kCw == 32, "column masks are 32-bit words");

// TMEM column of the bf16 operand slice kk (16 rows of K) once the element warps have packed
// their kCw fp32 columns into the first kCw/2 columns of the same range.
__host__ __device__ constexpr uint32_t packed_col(int kk) {
    return static_cast<uint32_t>(kCw * (kk / (kCw / 16)) + 8 * (kk % (kCw / 16)));
}
constexpr float kLog2e = 1.4426950408889634f;


// ----------------------------------------------------------------------- delta
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                    const __nv_bfloat16* __restrict__ d_o,
                                                    float* __restrict__ delta, int nq, int H,
                                                    int D, long long nrows) {
    // one row (token, head) per 16 threads, 8 channels per thread per step
    const long long row = (long long)blockIdx.x * 16 + threadIdx.x / 16;
    const int sub = threadIdx.x % 16;
    float acc = 0.f;
    if (row < nrows) {
        const __nv_bfloat16* a = o + row * D;
        const __nv_bfloat16* b = d_o + row * D;
        for (int c = sub * 8; c < D; c += 128) {
            const uint4 va = __ldg(reinterpret_cast<const uint4*>(a + c));
            const uint4 vb = __ldg(reinterpret_cast<const uint4*>(b + c));
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

constexpr int B_COUNT = 16;  // mbarrier slots reserved per CTA

// ===================================================================== dK / dV
// A dK/dV CTA walks the query blocks that see its keys, one 64-row query block at a time:
// Q and dO of a block are one TMA box each per 64 channels (16 KB for both halves of D),
// kept in kQst stages with their lse / Delta.
constexpr int kQst = 4;
constexpr uint32_t kQBlk = 64 * 128;   // bytes of one query block, one 64-channel half

struct DkdvPlan {
    uint32_t k, v, q, dq_o, lse, dl, grp_row, sub, bars, misc, total;
};

__host__ __device__ inline DkdvPlan dkdv_plan(int D, int S, int qb_total) {
    DkdvPlan p;
    const uint32_t nh = D / 64;
    p.k = 0;
    p.v = p.k + nh * kHalf;
    p.q = p.v + nh * kHalf;                 // kQst stages of one query block's Q
    p.dq_o = p.q + kQst * nh * kQBlk;       // kQst stages of its dO
    p.lse = p.dq_o + kQst * nh * kQBlk;     // kQst x 64 fp32 (log2 units, +inf = padding)
    p.dl = p.lse + kQst * 64 * 4;           // kQst x 64 fp32 Delta
    p.grp_row = p.dl + kQst * 64 * 4;       // 8*S
    p.sub = p.grp_row + 4u * 8u * S;        // query blocks that see the keys: qb << 2 | bits
    p.bars = (p.sub + 4u * qb_total + 7u) & ~7u;
    p.misc = p.bars + 8u * B_COUNT;
    p.total = p.misc + 4u * 8u;
    return p;
}

// Arguments of the backward launch: dQ CTAs and dK/dV CTAs share one grid (see bwd_kernel).
struct BwdKernelArgs {
    BwdArgs a;
    int n_pt_max;  // persistent key tiles per (b, h) of the dK/dV part
    int ucap;      // capacity of a query tile's local-block union
    int n_dq_x;    // dQ CTAs per (b, h): query tiles
    int n_kd_x;    // dK/dV CTAs per (b, h): persistent + local key tiles
};

// dK/dV of key tile cta_x of head h, batch b (body of bwd_kernel's dK/dV CTAs).
template <int D>
__device__ __forceinline__ void dkdv_body(const BwdKernelArgs& ka, const int cta_x, const int h, const int b) {
    constexpr int NH = D / 64;
    constexpr uint32_t TILE = NH * kHalf;
    constexpr uint32_t QSTAGE = NH * kQBlk;
    // TMEM: two buffers of (S^T | dP^T) for 64-query blocks (buffer x at 128 x, dP^T at +64),
    // then the dV and dK accumulators
    constexpr uint32_t kTmDV = 256, kTmDK = 256 + D;
    const BwdArgs& a = ka.a;
    const Geo& g = a.g;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int S = g.S;
    const int qb_total = a.q_frames / g.bt * g.nbf;
    const DkdvPlan PL = dkdv_plan(D, S, qb_total);
    uint8_t* sK = sm + PL.k;
    uint8_t* sV = sm + PL.v;
    uint8_t* sQ = sm + PL.q;
    uint8_t* sDO = sm + PL.dq_o;
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
    uint64_t* qd_empty = &bars[5];     // [kQst]
    uint64_t* sdp_full = &bars[9];     // [2] S^T and dP^T of a query block in TMEM buffer x
    uint64_t* pds_full = &bars[11];    // [2] P^T and dS^T written (one arrival per element warp)
    uint64_t* pass_done = &bars[13];   // dV/dK MMAs of the last query block done (one phase)
    uint64_t* drain = &bars[14];
    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kQst; ++s) {
            mbar_init(&qd_full[s], 1 + 32);  // producer expect_tx + 32 lse/Delta loaders
            mbar_init(&qd_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sdp_full[x], 1);
            mbar_init(&pds_full[x], kElemWarps);
        }
        mbar_init(pass_done, 1);
        mbar_init(drain, 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    if (g.brows < 64) zero_tiles(sm + PL.k, PL.lse - PL.k);
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
    // the query blocks that see these keys, in order, with bit kb set when the block selected
    // key block kb (persistent keys: every query block, both bits)
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
            if (bits) sub[base + __popc(m & ((1u << lane) - 1u))] = (qb << 2) | bits;
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
            if (lane == 0) {
                mbar_arrive_expect_tx(&qd_full[st], 2 * NH * box_bytes);
                const int f0 = b * a.q_frames + (qb / g.nbf) * g.bt;
                for (int hh = 0; hh < NH; ++hh) {
                    tma_load_5d(sQ + st * QSTAGE + hh * kQBlk, &a.tm_q, &qd_full[st], hh * 64, h, qbb.x0, qbb.y0, f0);
                    tma_load_5d(sDO + st * QSTAGE + hh * kQBlk, &a.tm_do, &qd_full[st], hh * 64, h, qbb.x0, qbb.y0, f0);
                }
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
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(128, 64, false, false);   // 128 keys x 64 queries
            constexpr uint32_t id_g = idesc_bf16(128, D, false, true);
            bool ok = mbar_wait(kv_full, 0, abort_flag, a.status);
            const uint32_t kb = smem_u32(sK), vb = smem_u32(sV);
            // S^T = K Q_u^T and dP^T = V dO_u^T of query block u into TMEM buffer u & 1; the
            // element warps turn them into P^T / dS^T (bf16, in place); dV += P^T dO_u and
            // dK += dS^T Q_u follow.  Issue order: block u + 2's S^T / dP^T right after block u's
            // dV / dK (the tensor pipe runs one thread's MMAs in issue order, so they never
            // overwrite P^T / dS^T before dV / dK have read them), which keeps the next block's
            // S^T / dP^T computing while the element warps work on the current one.
            auto issue_sdp = [&](int u) -> bool {
                const int st = u % kQst;
                if (!mbar_wait(&qd_full[st], (u / kQst) & 1, abort_flag, a.status)) return false;
                tc_fence_after();
                const uint32_t qs = smem_u32(sQ + st * QSTAGE), os = smem_u32(sDO + st * QSTAGE);
                const uint32_t buf = tmem + 128 * (u & 1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ka_ = (kk >> 2) * kHalf + (kk & 3) * 32;   // K / V tile: 128 rows
                    const uint32_t kq = (kk >> 2) * kQBlk + (kk & 3) * 32;    // Q / dO block: 64 rows
                    umma_ss(buf, sdesc_make(sdesc_lo(kb, 16) + (ka_ >> 4)), sdesc_make(sdesc_lo(qs, 16) + (kq >> 4)),
                            id_s, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ka_ = (kk >> 2) * kHalf + (kk & 3) * 32;
                    const uint32_t kq = (kk >> 2) * kQBlk + (kk & 3) * 32;
                    umma_ss(buf + 64, sdesc_make(sdesc_lo(vb, 16) + (ka_ >> 4)), sdesc_make(sdesc_lo(os, 16) + (kq >> 4)),
                            id_s, kk > 0);
                }
                umma_commit(&sdp_full[u & 1]);
                return true;
            };
            for (int u = 0; ok && u < min(2, n_sub); ++u) ok = issue_sdp(u);
            for (int u = 0; ok && u < n_sub; ++u) {
                const int st = u % kQst;
                if (!mbar_wait(&pds_full[u & 1], (u >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t qs = smem_u32(sQ + st * QSTAGE), os = smem_u32(sDO + st * QSTAGE);
                const uint32_t buf = tmem + 128 * (u & 1);
                // B operands dO / Q read MN-major: 64 channels per 128-byte row, the next 64
                // channels kQBlk bytes on, 16 query rows per MMA
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_ts(tmem + kTmDV, buf + 16 * kk, sdesc_make(sdesc_lo(os, kQBlk) + kk * 128), id_g,
                            (u > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_ts(tmem + kTmDK, buf + 64 + 16 * kk, sdesc_make(sdesc_lo(qs, kQBlk) + kk * 128), id_g,
                            (u > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&qd_empty[st]);
                // one phase, after the last block: the element warps may run two blocks ahead of
                // the dV/dK MMAs, so a per-block phase could not be waited on by parity alone
                if (u == n_sub - 1) umma_commit(pass_done);
                if (u + 2 < n_sub && !issue_sdp(u + 2)) { ok = false; break; }
            }
            if (!ok) {
                umma_commit(drain);
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else if (live && warp < kElemWarps) {
        // ------------------------------------------------------- element warps
        // warp w reads TMEM lanes 32 (w % 4).. (its key rows) and query columns
        // [16 (w / 4), +16) of the block's S^T / dP^T; it packs P^T / dS^T (bf16) into the
        // first 8 of those columns once it has read them, so no other warp's input is
        // overwritten.
        const int wq = warp & 3, cg = warp >> 2;
        const int r = 32 * wq + lane;
        const int c0 = 16 * cg;             // first query column of this warp
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
            tc_fence_after();
            const bool sel = key_valid && ((sub[u] >> kbr) & 1);
            const float l_mine = s_lse[st * 64 + c0 + (lane & 15)];
            const float d_mine = s_dl[st * 64 + c0 + (lane & 15)];
            const uint32_t buf = 128 * (u & 1);
            uint32_t pk[8], dk[8];
            {
                uint32_t sv[16], pv[16];
                tmem_ld16(tmem + lane_base + buf + c0, sv);
                tmem_ld16(tmem + lane_base + buf + 64 + c0, pv);
                tmem_ld_wait();
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    float ls[4], ds[4];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        ls[v] = __shfl_sync(0xffffffffu, l_mine, 4 * e4 + v);
                        ds[v] = __shfl_sync(0xffffffffu, d_mine, 4 * e4 + v);
                    }
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
            tmem_st8(tmem + lane_base + buf + c0, pk);
            tmem_st8(tmem + lane_base + buf + 64 + c0, dk);
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
            // channel chunks of 16: chunk c goes to element warp column group c % kNwq
            for (int c = cg; c < D / 16; c += kNwq) {
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
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ========================================================================== dQ
struct DqPlan {
    uint32_t q, dq_o, k, v, grp_row, tile_mask, uni_blk, uni_bits, blk_mask, bars, misc, total;
};

// dQ CTAs: K tiles live from S = Q K^T until the dQ MMA of their tile (three stages), V
// tiles only until dP = dO V^T (one stage).
constexpr int kDqKst = 3, kDqVst = 1;

__host__ __device__ inline DqPlan dq_plan(int D, int S, int ucap, int nbf) {
    DqPlan p;
    const uint32_t nh = D / 64;
    p.q = 0;
    p.dq_o = p.q + nh * kHalf;
    p.k = p.dq_o + nh * kHalf;
    p.v = p.k + kDqKst * nh * kHalf;
    p.grp_row = p.v + kDqVst * nh * kHalf;
    p.tile_mask = p.grp_row + 4u * 8u * S;              // [16-group tiles][4] valid key columns
    p.uni_blk = p.tile_mask + 16u * ((8u * S + 15u) / 16u);
    p.uni_bits = p.uni_blk + 4u * ucap;
    p.blk_mask = (p.uni_bits + 4u * ucap + 7u) & ~7u;  // [nbf] valid rows of each block
    p.bars = p.blk_mask + 8u * nbf;
    p.misc = p.bars + 8u * 16u;
    p.total = p.misc + 4u * 8u;
    return p;
}


// dQ of query tile `tile` of head h, batch b (body of bwd_kernel's dQ CTAs).
template <int D>
__device__ __forceinline__ void dq_body(const BwdKernelArgs& ka, const int tile, const int h, const int b) {
    constexpr int NH = D / 64;
    constexpr uint32_t TILE = NH * kHalf;
    // TMEM: two S buffers (tile t in buffer t & 1), dP, dQ
    constexpr uint32_t kTmS = 0, kTmP = 256, kTmQ = 384;
    const BwdArgs& a = ka.a;
    const Geo& g = a.g;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int S = g.S;
    const int ucap = ka.ucap;
    const DqPlan PL = dq_plan(D, S, ucap, g.nbf);
    uint8_t* sQ = sm + PL.q;
    uint8_t* sDO = sm + PL.dq_o;
    uint8_t* sK = sm + PL.k;
    uint8_t* sV = sm + PL.v;
    int32_t* grp_row = reinterpret_cast<int32_t*>(sm + PL.grp_row);
    uint32_t* tile_mask = reinterpret_cast<uint32_t*>(sm + PL.tile_mask);
    int32_t* uni_blk = reinterpret_cast<int32_t*>(sm + PL.uni_blk);
    int32_t* uni_bits = reinterpret_cast<int32_t*>(sm + PL.uni_bits);
    uint64_t* blk_mask = reinterpret_cast<uint64_t*>(sm + PL.blk_mask);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL.bars);
    int* misc = reinterpret_cast<int*>(sm + PL.misc);
    volatile int* abort_flag = misc + 1;
    uint64_t* q_full = &bars[0];
    uint64_t* k_full = &bars[1];    // [kDqKst]
    uint64_t* k_empty = &bars[4];   // [kDqKst]
    uint64_t* v_full = &bars[7];
    uint64_t* v_empty = &bars[8];
    uint64_t* sdp_full = &bars[9];  // S and dP of a tile computed
    uint64_t* dp_free = &bars[10];  // every element warp has read dP (kElemWarps arrivals)
    uint64_t* ds_full = &bars[11];  // dS written (kElemWarps arrivals)
    uint64_t* dq_done = &bars[12];
    uint64_t* drain = &bars[13];

    const int bh = b * g.H + h;
    const int qb_total = a.q_frames / g.bt * g.nbf;
    const int nq = a.q_frames * g.tf;
    const int qb0 = 2 * tile;
    const int qb1 = (2 * tile + 1 < qb_total) ? 2 * tile + 1 : -1;
    const int nl = a.local_frames / g.bt * g.nbf;
    const uint32_t box_bytes = static_cast<uint32_t>(g.brows) * 128u;  // one block, one 64-channel half
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kDqKst; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        mbar_init(v_full, 1);
        mbar_init(v_empty, 1);
        mbar_init(sdp_full, 1);
        mbar_init(dp_free, kElemWarps);
        mbar_init(ds_full, kElemWarps);
        mbar_init(dq_done, 1);
        mbar_init(drain, 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < g.nbf; i += blockDim.x) blk_mask[i] = block_rows_mask(g, i);
    if (g.brows < 64) zero_tiles(sm + PL.q, PL.grp_row - PL.q);
    if (warp == kMmaWarp) tmem_alloc(reinterpret_cast<uint32_t*>(misc + 0), 512);
    if (warp == 0) {
        const int G = build_groups(a.pers_len, bh, S, grp_row, a.status);
        if (lane == 0) misc[2] = G;
        __syncwarp();
        // valid key columns of each 16-group tile, one 32-bit word per 4 groups
        for (int w = lane; w < 4 * ((G + 15) / 16); w += 32) {
            uint32_t m = 0;
            for (int gq = 0; gq < 4; ++gq) {
                const int gi = 4 * w + gq;
                if (gi < G) {
                    const int nv = group_rows(grp_row[gi]);
                    m |= (nv >= 8 ? 0xffu : ((1u << nv) - 1u)) << (8 * gq);
                }
            }
            tile_mask[w] = m;
        }
    }
    if (warp == 1 && lane == 0) {
        const int c0 = min(max(a.cnt[(size_t)bh * qb_total + qb0], 0), a.idx_stride);
        const int c1 = qb1 >= 0 ? min(max(a.cnt[(size_t)bh * qb_total + qb1], 0), a.idx_stride) : 0;
        const int32_t* i0 = a.idx + ((size_t)bh * qb_total + qb0) * a.idx_stride;
        const int32_t* i1 = a.idx + ((size_t)bh * qb_total + (qb1 >= 0 ? qb1 : qb0)) * a.idx_stride;
        int p = 0, q = 0, u = 0;
        while (p < c0 || q < c1) {
            if (u == ucap) {
                set_status(a.status, PBSA_ERR_DEVICE_CHECK);
                break;
            }
            const int v0 = p < c0 ? i0[p] : 0x7fffffff;
            const int v1 = q < c1 ? i1[q] : 0x7fffffff;
            int blk, bits;
            if (v0 == v1) {
                blk = v0; bits = 3; ++p; ++q;
            } else if (v0 < v1) {
                blk = v0; bits = 1; ++p;
            } else {
                blk = v1; bits = 2; ++q;
            }
            if (blk < 0 || blk >= nl) {
                set_status(a.status, PBSA_ERR_DEVICE_CHECK);
                continue;
            }
            uni_blk[u] = blk;
            uni_bits[u] = bits;
            ++u;
        }
        misc[3] = u;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(misc[0]);
    const int G = misc[2], U = misc[3];
    const int n_pt = (G + 15) / 16;
    const int n_tiles = n_pt + (U + 1) / 2;

    if (warp == kProdWarp) {
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, 2 * 2 * NH * box_bytes);
            for (int hb = 0; hb < 2; ++hb) {
                const int qb = (hb == 1 && qb1 >= 0) ? qb1 : qb0;
                const BlockBox qbb = block_box(g, qb % g.nbf);
                const int f0 = b * a.q_frames + (qb / g.nbf) * g.bt;
                for (int hh = 0; hh < NH; ++hh) {
                    tma_load_5d(sQ + hh * kHalf + hb * (kHalf / 2), &a.tm_q, q_full, hh * 64, h, qbb.x0, qbb.y0, f0);
                    tma_load_5d(sDO + hh * kHalf + hb * (kHalf / 2), &a.tm_do, q_full, hh * 64, h, qbb.x0, qbb.y0, f0);
                }
            }
            // K of tile it into stage it % 3 once the dQ MMA of tile it - 3 is done; V of tile
            // it into the single V stage once dP of tile it - 1 is done
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int st = it % kDqKst;
                if (it >= kDqKst && !mbar_wait(&k_empty[st], ((it / kDqKst) - 1) & 1, abort_flag, a.status)) break;
                uint8_t* dk = sK + st * TILE;
                const uint32_t tile_bytes = it < n_pt ? TILE : 2 * NH * box_bytes;
                mbar_arrive_expect_tx(&k_full[st], tile_bytes);
                if (it < n_pt) {
                    tma_load_groups16<NH>(dk, kHalf, &a.tm_kp, &a.tm_kp64, grp_row, it * 16, G, &k_full[st]);
                } else {
                    const int j = it - n_pt;
                    for (int hb = 0; hb < 2; ++hb) {
                        const int L = uni_blk[min(2 * j + hb, U - 1)];
                        const BlockBox kbb = block_box(g, L % g.nbf);
                        const int fr = b * g.W + (a.ring_head + (L / g.nbf) * g.bt) % g.W;
                        for (int hh = 0; hh < NH; ++hh)
                            tma_load_5d(dk + hh * kHalf + hb * (kHalf / 2), &a.tm_kl, &k_full[st], hh * 64, h,
                                        kbb.x0, kbb.y0, fr);
                    }
                }
                if (it >= 1 && !mbar_wait(v_empty, (it - 1) & 1, abort_flag, a.status)) { ++issued; break; }
                mbar_arrive_expect_tx(v_full, tile_bytes);
                if (it < n_pt) {
                    tma_load_groups16<NH>(sV, kHalf, &a.tm_vp, &a.tm_vp64, grp_row, it * 16, G, v_full);
                } else {
                    const int j = it - n_pt;
                    for (int hb = 0; hb < 2; ++hb) {
                        const int L = uni_blk[min(2 * j + hb, U - 1)];
                        const BlockBox kbb = block_box(g, L % g.nbf);
                        const int fr = b * g.W + (a.ring_head + (L / g.nbf) * g.bt) % g.W;
                        for (int hh = 0; hh < NH; ++hh)
                            tma_load_5d(sV + hh * kHalf + hb * (kHalf / 2), &a.tm_vl, v_full, hh * 64, h,
                                        kbb.x0, kbb.y0, fr);
                    }
                }
                ++issued;
            }
            if (*abort_flag) {
                // let the copies already issued land before the CTA leaves
                mbar_wait_drain(q_full, 0, 100000000ull);
                for (int it = max(0, issued - kDqKst); it < issued; ++it)
                    mbar_wait_drain(&k_full[it % kDqKst], (it / kDqKst) & 1, 100000000ull);
                if (issued > 0) mbar_wait_drain(v_full, (issued - 1) & 1, 100000000ull);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
            constexpr uint32_t id_g = idesc_bf16(128, D, false, true);
            bool ok = mbar_wait(q_full, 0, abort_flag, a.status);
            const uint32_t qbase = smem_u32(sQ), obase = smem_u32(sDO), vb = smem_u32(sV);
            // S(t) = Q K(t)^T into S buffer t & 1; dP(t) = dO V(t)^T; both then committed to
            // sdp_full.  Per tile t the issue order is S(t+1), dP(t+1), dQ += dS(t) K(t): the
            // next tile's S and dP run while the element warps work on tile t (dP(t+1) only once
            // every element warp has read dP(t)); the tensor pipe executes one thread's MMAs in
            // issue order, so S(t+2) never overwrites dS(t) before dQ(t) has read it.
            auto issue_s = [&](int t) -> bool {
                const int st = t % kDqKst;
                if (!mbar_wait(&k_full[st], (t / kDqKst) & 1, abort_flag, a.status)) return false;
                tc_fence_after();
                const uint32_t kb = smem_u32(sK + st * TILE);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                    umma_ss(tmem + kTmS + 128 * (t & 1), sdesc_make(sdesc_lo(qbase, 16) + (off >> 4)),
                            sdesc_make(sdesc_lo(kb, 16) + (off >> 4)), id_s, kk > 0);
                }
                return true;
            };
            auto issue_dp = [&](int t) -> bool {
                if (!mbar_wait(v_full, t & 1, abort_flag, a.status)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                    umma_ss(tmem + kTmP, sdesc_make(sdesc_lo(obase, 16) + (off >> 4)),
                            sdesc_make(sdesc_lo(vb, 16) + (off >> 4)), id_s, kk > 0);
                }
                umma_commit(v_empty);
                umma_commit(sdp_full);
                return true;
            };
            if (ok && n_tiles > 0) ok = issue_s(0) && issue_dp(0);
            for (int it = 0; ok && it < n_tiles; ++it) {
                if (it + 1 < n_tiles) {
                    if (!issue_s(it + 1)) { ok = false; break; }
                    if (!mbar_wait(dp_free, it & 1, abort_flag, a.status)) { ok = false; break; }
                    if (!issue_dp(it + 1)) { ok = false; break; }
                }
                if (!mbar_wait(ds_full, it & 1, abort_flag, a.status)) { ok = false; break; }
                tc_fence_after();
                const int st = it % kDqKst;
                const uint32_t kb = smem_u32(sK + st * TILE);
                const uint32_t s_buf = tmem + kTmS + 128 * (it & 1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tmem + kTmQ, s_buf + packed_col(kk), sdesc_make(sdesc_lo(kb, kHalf) + kk * 128), id_g,
                            (it > 0 || kk > 0) ? 1u : 0u);
                // one phase, after the last tile: the element warps may finish a tile before the
                // previous tile's dQ MMAs are even issued, so a per-tile phase could not be waited
                // on by parity alone
                if (it == n_tiles - 1) umma_commit(dq_done);
                umma_commit(&k_empty[st]);
            }
            if (!ok) {
                umma_commit(drain);
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else if (warp < kElemWarps) {
        // element warps: warp w owns query rows 32 (w % 4).. (TMEM lanes) and key columns
        // [32 (w / 4), +32) of S / dP; it packs dS (bf16) into the first 16 of them
        const int wq = warp & 3, cg = warp >> 2;
        const int r = 32 * wq + lane;
        const int c0 = kCw * cg;              // first key column of this warp
        const int kh = c0 >> 6;               // key block (half of a local key tile) of those columns
        const int hq = r >> 6;
        const int qbr = hq ? qb1 : qb0;
        const int qbv = qbr >= 0 ? qbr : qb0;
        const BlockBox qbb = block_box(g, qbv % g.nbf);
        int qt, qy, qx;
        const bool row_valid = block_row(g, qbb, r & 63, &qt, &qy, &qx) && qbr >= 0;
        const size_t tok = (size_t)((qbv / g.nbf) * g.bt + qt) * g.tf + (qbb.y0 + qy) * g.fw + qbb.x0 + qx;
        const float lse2 = row_valid ? a.lse[(size_t)bh * nq + tok] * kLog2e : CUDART_INF_F;
        const float dl = row_valid ? a.delta[(size_t)bh * nq + tok] : 0.f;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const float sl2 = kLog2e / sqrtf(static_cast<float>(D));
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.status));
        };
        bool ok = true;
        for (int it = 0; it < n_tiles; ++it) {
            if (!wwait(sdp_full, it & 1)) { ok = false; break; }
            tc_fence_after();
            // valid-column mask of this warp's 32 key columns
            uint32_t vmask;
            if (it < n_pt) {
                vmask = tile_mask[4 * it + cg];   // the warp's 32 columns: groups 16 it + 4 cg ..
            } else {
                const int u = 2 * (it - n_pt) + kh;
                const bool has = u < U;
                const int L = uni_blk[has ? u : 0];
                const bool sel = has && ((uni_bits[has ? u : 0] >> hq) & 1);
                // columns c0.. are the block's box rows (c0 & 63) + e
                vmask = sel ? static_cast<uint32_t>(blk_mask[L % g.nbf] >> (c0 & 63)) : 0u;
            }
            // dP first: once every element warp holds its dP columns the MMA thread may
            // compute the next tile's dP into the same columns
            const uint32_t s_buf = kTmS + 128 * (it & 1);
            float dpm[kCw];
            {
                uint32_t pv[kCw];
                tmem_ld16(tmem + lane_base + kTmP + c0, *reinterpret_cast<uint32_t(*)[16]>(pv));
                tmem_ld16(tmem + lane_base + kTmP + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(pv + 16));
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < kCw; ++e) dpm[e] = __uint_as_float(pv[e]) - dl;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dp_free);
            uint32_t dk[kCw / 2];
#pragma unroll
            for (int sc = 0; sc < kCw / 16; ++sc) {
                uint32_t sv[16];
                tmem_ld16(tmem + lane_base + s_buf + c0 + 16 * sc, sv);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    float dsv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const bool valid = (vmask >> (16 * sc + e + u)) & 1u;
                        const float p = valid ? fast_exp2(__uint_as_float(sv[e + u]) * sl2 - lse2) : 0.f;
                        dsv[u] = p * dpm[16 * sc + e + u];
                    }
                    dk[8 * sc + e / 2] = pack_bf16x2(dsv[0], dsv[1]);
                }
            }
            tmem_st16(tmem + lane_base + s_buf + c0, dk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full);
        }
        ok = named_bar_and(2, 32 * kElemWarps, ok);
        if (ok && n_tiles > 0) {
            ok = named_bar_and(2, 32 * kElemWarps, wwait(dq_done, 0));
            tc_fence_after();
        }
        if (ok) {
            const float isd = 1.0f / sqrtf(static_cast<float>(D));
            float* dst = a.dq + (((size_t)b * nq + tok) * g.H + h) * D;
            for (int c = cg; c < D / 16; c += kNwq) {
                uint32_t v[16];
                if (n_tiles > 0) {
                    tmem_ld16(tmem + lane_base + kTmQ + 16 * c, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = 0u;
                }
                if (row_valid) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(dst + 16 * c + e) =
                            make_float4(__uint_as_float(v[e]) * isd, __uint_as_float(v[e + 1]) * isd,
                                        __uint_as_float(v[e + 2]) * isd, __uint_as_float(v[e + 3]) * isd);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// One grid for both gradient kernels, dQ CTAs first: they are the long ones (a query tile
// against its whole key stream), so the many short dK/dV CTAs that follow fill the SMs the
// last dQ wave leaves idle instead of starting after it.  The two parts are independent
// (they only read the forward's tensors and Delta and write different outputs).
template <int D>
__global__ void __launch_bounds__(kThreads, 1) bwd_kernel(const __grid_constant__ BwdKernelArgs ka) {
    const int H = ka.a.g.H;
    const int n_dq = ka.n_dq_x * H * ka.a.g.B;
    int i = blockIdx.x;
    if (i < n_dq) {
        const int r = i / ka.n_dq_x;
        dq_body<D>(ka, i % ka.n_dq_x, r % H, r / H);
    } else {
        i -= n_dq;
        const int r = i / ka.n_kd_x;
        dkdv_body<D>(ka, i % ka.n_kd_x, r % H, r / H);
    }
}

template <class K, class A>
cudaError_t launch_k(K kernel, const A& args, dim3 grid, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, st>>>(args);
    return cudaGetLastError();
}

}  // namespace

size_t attn_bwd_smem_bytes(const Geo& g, int q_frames, int ucap) {
    const size_t a = dkdv_plan(g.D, g.S, q_frames / g.bt * g.nbf).total + 1024;
    const size_t b = dq_plan(g.D, g.S, ucap, g.nbf).total + 1024;
    size_t m = a > b ? a : b;
    return m < 120 * 1024 ? 120 * 1024 : m;
}

cudaError_t launch_attn_bwd(const BwdArgs& a, cudaStream_t st) {
    const Geo& g = a.g;
    const int nq = a.q_frames * g.tf;
    const long long nrows = (long long)g.B * nq * g.H;
    delta_kernel<<<(unsigned)((nrows + 15) / 16), 256, 0, st>>>(a.out, a.dout, a.delta, nq, g.H, g.D, nrows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    const int qb_total = a.q_frames / g.bt * g.nbf;
    BwdKernelArgs ka;
    ka.a = a;
    ka.n_pt_max = (g.S * 8 + 15) / 16;
    ka.ucap = a.ucap;
    ka.n_dq_x = (qb_total + 1) / 2;
    ka.n_kd_x = ka.n_pt_max + (a.local_frames / g.bt * g.nbf + 1) / 2;
    const size_t smem = attn_bwd_smem_bytes(g, a.q_frames, a.ucap);
    const long long ctas = (long long)(ka.n_dq_x + ka.n_kd_x) * g.H * g.B;
    if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)ctas);
    return g.D == 128 ? launch_k(bwd_kernel<128>, ka, grid, smem, st)
                      : launch_k(bwd_kernel<64>, ka, grid, smem, st);
}

}  // namespace pbsa
