// attn_fwd.cu - PBSA forward on sm_100a (TMA + tcgen05 + TMEM).
//
// Sparse Forcing (pith.science abstract; project page kernel features): every query token
// attends to all blocks of the persistent cache and to the top-k blocks of the local
// window selected for its query block, with softmax scale 1/sqrt(D).  With a mass output
// the kernel also accumulates, per persistent slot and per local block, the softmax
// probability summed over the chunk's query rows (the score that ranks blocks when the
// window slides).
//
// One CTA = four query blocks of one (batch, head), split into two 128-row query tiles
// ("sides" A and B, two blocks each; a block is one 5-D TMA box of bt x bh x bw tokens
// placed in a 64-row half of the tile, rows past bt*bh*bw zero; ragged edge blocks are
// zero-filled on load and clipped on store).  Key tiles are 128 keys:
//   * persistent tiles (shared by both sides): the occupied slots' rows compacted into a
//     stream of 8-row groups (ceil(len / 8) groups per slot; the last group of a slot whose
//     length is not a multiple of 8 is partly valid and its other rows are masked), 16
//     groups per tile, loaded as one 64-row TMA box wherever eight groups are contiguous
//     rows (a full slot);
//   * local tiles (one side each): the union of that side's two selections, two key blocks
//     per tile (one per 64-row half); columns the row's query block did not select, or
//     outside the block or the frame, are masked.  A-tiles and B-tiles alternate.
// TMEM (512 columns): S_A | S_B | O_A | O_B.  P (bf16) is written over the first 64 columns
// of its S and read by a TS MMA; the tensor pipe executes one thread's MMAs in issue order,
// so S = Q K^T of a side's next tile may be issued right after the O += P V that reads
// its P.  Issue order per persistent tile: QK_A(t), PV_B(t-1), QK_B(t), PV_A(t), so each
// side's softmax of tile t runs while the other side's MMAs occupy the tensor pipe.
// Warp roles (384 threads): warps 0-3 softmax of side A, 4-7 side B (one query row per
// thread), warp 8 K (and Q) producer, warp 9 V producer, warp 10 MMA issuer, warp 11 idle.  K and V
// stages have separate full/empty barriers.  O is rescaled only when a row maximum grows by
// more than 2^8; so the softmax first exponentiates half of the row against the running
// reference while taking the tile's row maximum in the same pass, and only a warp with a
// row that needs a new reference rescales O and redoes that half from S (still intact in
// TMEM).  Each half's P is stored as soon as it is packed.  Mass: each row emits, per
// slot/block it saw, log2 of its partial
// probability sum (relative to its running maximum) into workspace; once the final
// log-sum-exp is known the side converts them, sums over its rows and adds one value per
// slot/block to the global mass arrays.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

constexpr int kNst = 2;                // K and V pipeline stages
constexpr uint32_t kHalf = 128 * 128;  // bytes of 128 rows x 64 bf16 channels
constexpr uint32_t kTmCols = 512;
constexpr int kThreads = 384;
// Register split: the kernel launches at kLaunchRegs per thread (384 x 168 = 64512); the
// producer/MMA warpgroup drops to kRegsIo and both softmax warpgroups rise to kRegsSoftmax,
// 2 x 128 x 216 + 128 x 72 = 64512, exactly the launch pool.  The host refuses to launch if
// ptxas did not give the kernel kLaunchRegs, so the increase can always be satisfied.
constexpr int kLaunchRegs = 168, kRegsIo = 72, kRegsSoftmax = 216;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsIo <= kThreads * kLaunchRegs, "register split");
constexpr float kLog2e = 1.4426950408889634f;

struct SmemPlan {
    uint32_t q, k, v, grp_row, grp_seg, seg_slot, tile_end, tile_seg, tile_mask, uni_blk, uni_bits,
        lse_s, blk_mask, bars, misc, total;
};

__host__ __device__ inline SmemPlan fwd_plan(int D, int S, int ucap, int nbf) {
    SmemPlan p;
    const uint32_t nh = D / 64;
    const uint32_t n_pt_max = (8u * S + 15u) / 16u;
    p.q = 0;                                 // 2 sides
    p.k = p.q + 2 * nh * kHalf;
    p.v = p.k + kNst * nh * kHalf;
    p.grp_row = p.v + kNst * nh * kHalf;
    p.grp_seg = p.grp_row + 4u * 8u * S;
    p.seg_slot = p.grp_seg + 4u * 8u * S;
    p.tile_end = p.seg_slot + 4u * S;        // per persistent tile: groups that end a slot
    p.tile_seg = p.tile_end + 4u * n_pt_max; // per persistent tile: slot rank of group 0
    p.tile_mask = p.tile_seg + 4u * n_pt_max; // per persistent tile: 128-bit valid-column mask
    p.uni_blk = p.tile_mask + 16u * n_pt_max; // [2][ucap]
    p.uni_bits = p.uni_blk + 8u * ucap;      // [2][ucap]
    p.lse_s = p.uni_bits + 8u * ucap;        // [2][128] row log-sum-exp (log2) for the mass
    p.blk_mask = (p.lse_s + 2u * 128u * 4u + 7u) & ~7u;  // [nbf] valid rows of each block
    p.bars = p.blk_mask + 8u * nbf;
    p.misc = p.bars + 8u * 24u;
    p.total = p.misc + 4u * 16u;
    return p;
}

// barrier slots
enum {
    B_Q = 0, B_KF = 1, B_KE = 3, B_VF = 5, B_VE = 7, B_SF = 9, B_PF = 11, B_PV = 13, B_DRAIN = 15
};
// misc slots
enum { M_TMEM = 0, M_ABORT = 1, M_G = 2, M_OCC = 3, M_UA = 4, M_UB = 5 };

struct FwdKernelArgs {
    FwdArgs a;
    int n_groups;  // CTAs per (b, h): ceil(QB / 4)
};


__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (a.x * s - m, a.y * s - m) on the packed fp32x2 pipe
__device__ __forceinline__ float2 ffma2(float2 a, float s, float m) {
    uint64_t r;
    const uint64_t av = (static_cast<uint64_t>(__float_as_uint(a.y)) << 32) | __float_as_uint(a.x);
    const uint64_t sv = (static_cast<uint64_t>(__float_as_uint(s)) << 32) | __float_as_uint(s);
    const uint64_t mv = (static_cast<uint64_t>(__float_as_uint(-m)) << 32) | __float_as_uint(-m);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(av), "l"(sv), "l"(mv));
    return make_float2(__uint_as_float(static_cast<uint32_t>(r)), __uint_as_float(static_cast<uint32_t>(r >> 32)));
}

// exp_half<0> plus the maximum of all 128 raw values, read before they are overwritten:
// the ALU max work interleaves with the MUFU exponentials.
__device__ __forceinline__ float exp_half0_max(float (&x)[128], float sl2, float mu, float (&gs)[16]) {
    float mx[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) mx[j] = -CUDART_INF_F;
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) {
#pragma unroll
        for (int j = 0; j < 8; j += 2) mx[j / 2] = max3f(mx[j / 2], x[8 * gq + j], x[8 * gq + j + 1]);
#pragma unroll
        for (int j = 0; j < 8; j += 2) mx[4 + j / 2] = max3f(mx[4 + j / 2], x[64 + 8 * gq + j], x[64 + 8 * gq + j + 1]);
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
            const int c = 8 * gq + 2 * pr;
            const float2 q = ffma2(make_float2(x[c], x[c + 1]), sl2, mu);
            x[c] = fast_exp2(q.x);
            x[c + 1] = fast_exp2(q.y);
        }
        gs[gq] = ((x[8 * gq + 0] + x[8 * gq + 1]) + (x[8 * gq + 2] + x[8 * gq + 3])) +
                 ((x[8 * gq + 4] + x[8 * gq + 5]) + (x[8 * gq + 6] + x[8 * gq + 7]));
    }
    return max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// p = 2^(x * sl2 - mu) over the 64 columns [64 H, 64 H + 64) of a row, in place, with their
// 8-column group sums.
template <int H>
__device__ __forceinline__ void exp_half(float (&x)[128], float sl2, float mu, float (&gs)[16]) {
#pragma unroll
    for (int gq = 8 * H; gq < 8 * H + 8; ++gq) {
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
            const int c = 8 * gq + 2 * pr;
            const float2 q = ffma2(make_float2(x[c], x[c + 1]), sl2, mu);
            x[c] = fast_exp2(q.x);
            x[c + 1] = fast_exp2(q.y);
        }
        gs[gq] = ((x[8 * gq + 0] + x[8 * gq + 1]) + (x[8 * gq + 2] + x[8 * gq + 3])) +
                 ((x[8 * gq + 4] + x[8 * gq + 5]) + (x[8 * gq + 6] + x[8 * gq + 7]));
    }
}

// Consumers of stream tile t: bit 0 = side A, bit 1 = side B; *lj = local tile index.
// Persistent tiles come first (both sides), then the sides' local tiles alternate A, B.
__device__ __forceinline__ int tile_cons(int t, int n_pt, int nla, int nlb, bool has_b, int* lj) {
    if (t < n_pt) {
        *lj = -1;
        return has_b ? 3 : 1;
    }
    const int j = t - n_pt, m = min(nla, nlb);
    if (j < 2 * m) {
        *lj = j >> 1;
        return (j & 1) ? 2 : 1;
    }
    *lj = m + (j - 2 * m);
    return nla > nlb ? 1 : 2;
}

template <int D, bool MASS>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdKernelArgs ka) {
    constexpr int NH = D / 64;
    constexpr uint32_t KV_BYTES = NH * kHalf;
    constexpr uint32_t Q_SIDE = NH * kHalf;
    const FwdArgs& a = ka.a;
    const Geo& g = a.g;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int S = g.S;
    const int ucap = a.ucap;
    const SmemPlan P = fwd_plan(D, S, ucap, g.nbf);
    uint8_t* sQ = sm + P.q;
    uint8_t* sK = sm + P.k;
    uint8_t* sV = sm + P.v;
    int32_t* grp_row = reinterpret_cast<int32_t*>(sm + P.grp_row);
    int32_t* grp_seg = reinterpret_cast<int32_t*>(sm + P.grp_seg);
    int32_t* seg_slot = reinterpret_cast<int32_t*>(sm + P.seg_slot);
    uint32_t* tile_end = reinterpret_cast<uint32_t*>(sm + P.tile_end);
    int32_t* tile_seg = reinterpret_cast<int32_t*>(sm + P.tile_seg);
    uint4* tile_mask = reinterpret_cast<uint4*>(sm + P.tile_mask);
    int32_t* uni_blk = reinterpret_cast<int32_t*>(sm + P.uni_blk);
    int32_t* uni_bits = reinterpret_cast<int32_t*>(sm + P.uni_bits);
    float* lse_s = reinterpret_cast<float*>(sm + P.lse_s);
    uint64_t* blk_mask = reinterpret_cast<uint64_t*>(sm + P.blk_mask);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P.bars);
    int* misc = reinterpret_cast<int*>(sm + P.misc);
    volatile int* abort_flag = misc + M_ABORT;

    const int grp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * g.H + h;
    const int qb_total = a.q_frames / g.bt * g.nbf;
    const int nl = a.local_frames / g.bt * g.nbf;
    const int head_g = a.ring_head / g.bt;          // ring frame group of window group 0
    const uint32_t box_bytes = static_cast<uint32_t>(g.brows) * 128u;  // one block, one 64-channel half
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // query blocks of the two sides (-1 = none)
    auto qblock = [&](int X, int i) -> int {
        const int qb = 4 * grp + 2 * X + i;
        return qb < qb_total ? qb : -1;
    };
    const bool has_b = qblock(1, 0) >= 0;

    // ------------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        mbar_init(&bars[B_Q], 1);
        for (int s = 0; s < kNst; ++s) {
            mbar_init(&bars[B_KF + s], 1);
            mbar_init(&bars[B_KE + s], 1);
            mbar_init(&bars[B_VF + s], 1);
            mbar_init(&bars[B_VE + s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars[B_SF + x], 1);
            mbar_init(&bars[B_PF + x], 128);
            mbar_init(&bars[B_PV + x], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        misc[M_ABORT] = 0;
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < g.nbf; i += blockDim.x) blk_mask[i] = block_rows_mask(g, i);
    if (g.brows < 64) {
        // rows past a block's box are never written by TMA: zero every Q/K/V tile once so
        // that they hold finite values (masked columns multiply them by exact zeros)
        uint4* z = reinterpret_cast<uint4*>(sm + P.q);
        const int n16 = static_cast<int>((P.grp_row - P.q) / 16);
        for (int e = threadIdx.x; e < n16; e += blockDim.x) z[e] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == 10) tmem_alloc(reinterpret_cast<uint32_t*>(misc + M_TMEM), kTmCols);
    if (warp == 0) {
        // compacted stream of the occupied slots' 8-row groups; a group's entry is its first
        // row in the slot store with (valid rows & 7) in the low 3 bits (0 = all 8 valid)
        int run = 0, occ = 0;
        for (int s0 = 0; s0 < S; s0 += 32) {
            const int s = s0 + lane;
            int len = (s < S) ? a.pers_len[(size_t)bh * S + s] : 0;
            if (len < 0 || len > 64) {
                set_status(a.status, PBSA_ERR_DEVICE_CHECK);
                len = 0;
            }
            const int ng = (len + 7) >> 3, oc = ng > 0 ? 1 : 0;
            int inc_g = ng, inc_o = oc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int vg = __shfl_up_sync(0xffffffffu, inc_g, o);
                const int vo = __shfl_up_sync(0xffffffffu, inc_o, o);
                if (lane >= o) {
                    inc_g += vg;
                    inc_o += vo;
                }
            }
            const int gstart = run + inc_g - ng, rank = occ + inc_o - oc;
            if (ng > 0) {
                seg_slot[rank] = s;
                for (int i = 0; i < ng; ++i) {
                    grp_row[gstart + i] = (((bh * S) + s) * 64 + 8 * i) | (min(8, len - 8 * i) & 7);
                    grp_seg[gstart + i] = rank;
                }
            }
            run += __shfl_sync(0xffffffffu, inc_g, 31);
            occ += __shfl_sync(0xffffffffu, inc_o, 31);
        }
        if (lane == 0) {
            misc[M_G] = run;
            misc[M_OCC] = occ;
        }
        __syncwarp();
        // per 16-group tile: bit g set when group g is the last group of its slot, and the
        // valid key columns (8 per group, fewer in a slot's partial last group, none past G)
        for (int t = lane; t * 16 < run; t += 32) {
            uint32_t ends = 0;
            uint32_t mw[4] = {0u, 0u, 0u, 0u};
            for (int gq = 0; gq < 16; ++gq) {
                const int gi = 16 * t + gq;
                if (gi < run && (gi + 1 == run || grp_seg[gi + 1] != grp_seg[gi])) ends |= 1u << gq;
                if (gi < run) {
                    const int nv = grp_row[gi] & 7;
                    mw[gq >> 2] |= (nv ? ((1u << nv) - 1u) : 0xffu) << (8 * (gq & 3));
                }
            }
            tile_end[t] = ends;
            tile_seg[t] = grp_seg[16 * t];
            tile_mask[t] = make_uint4(mw[0], mw[1], mw[2], mw[3]);
        }
    }
    if ((warp == 1 || warp == 2) && lane == 0) {
        // union of one side's two selections (both lists ascending)
        const int X = warp - 1;
        const int q0 = qblock(X, 0), q1 = qblock(X, 1);
        int u = 0;
        if (q0 >= 0) {
            const int c0 = min(max(a.cnt[(size_t)bh * qb_total + q0], 0), a.idx_stride);
            const int c1 = q1 >= 0 ? min(max(a.cnt[(size_t)bh * qb_total + q1], 0), a.idx_stride) : 0;
            const int32_t* i0 = a.idx + ((size_t)bh * qb_total + q0) * a.idx_stride;
            const int32_t* i1 = a.idx + ((size_t)bh * qb_total + (q1 >= 0 ? q1 : q0)) * a.idx_stride;
            int p = 0, q = 0;
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
                uni_blk[X * ucap + u] = blk;
                uni_bits[X * ucap + u] = bits;
                ++u;
            }
        }
        misc[M_UA + X] = u;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = static_cast<uint32_t>(misc[M_TMEM]);
    const int G = misc[M_G], n_occ = misc[M_OCC];
    const int UA = misc[M_UA], UB = misc[M_UB];
    const int n_pt = (G + 15) / 16;
    const int nla = (UA + 1) / 2, nlb = has_b ? (UB + 1) / 2 : 0;
    const int n_stream = n_pt + nla + nlb;
    const int n_side0 = n_pt + nla, n_side1 = has_b ? n_pt + nlb : 0;

    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsIo));
      if (warp == 8 || warp == 9) {
        // ------------------------------------------------- TMA producers (K+Q, V)
        // the whole warp runs this; one elected lane issues each copy and barrier arrival
        {
            auto one = [&](auto&& f) {
                if (elect_one()) f();
                __syncwarp();
            };
            const bool isK = warp == 8;
            const CUtensorMap* mp = isK ? &a.tm_kp : &a.tm_vp;
            const CUtensorMap* mp64 = isK ? &a.tm_kp64 : &a.tm_vp64;
            const CUtensorMap* ml = isK ? &a.tm_kl : &a.tm_vl;
            uint8_t* base = isK ? sK : sV;
            uint64_t* full = &bars[isK ? B_KF : B_VF];
            uint64_t* empty = &bars[isK ? B_KE : B_VE];
            one([&] {
                tma_prefetch_desc(mp);
                tma_prefetch_desc(mp64);
                tma_prefetch_desc(ml);
            });
            if (isK) {
                one([&] {
                    tma_prefetch_desc(&a.tm_q);
                    mbar_arrive_expect_tx(&bars[B_Q], 2 * 2 * NH * box_bytes);
                });
                for (int X = 0; X < 2; ++X)
                    for (int hb = 0; hb < 2; ++hb) {
                        int qb = qblock(X, hb);
                        if (qb < 0) qb = qblock(0, 0);  // filler rows, never stored
                        const BlockBox qbb = block_box(g, qb % g.nbf);
                        const int f0 = b * a.q_frames + (qb / g.nbf) * g.bt;
                        for (int hh = 0; hh < NH; ++hh)
                            one([&] {
                                tma_load_5d(sQ + X * Q_SIDE + hh * kHalf + hb * (kHalf / 2), &a.tm_q, &bars[B_Q],
                                            hh * 64, h, qbb.x0, qbb.y0, f0);
                            });
                    }
            }
            int issued = 0;
            for (int t = 0; t < n_stream; ++t) {
                const int st = t % kNst;
                if (t >= kNst &&
                    !__all_sync(0xffffffffu, mbar_wait(&empty[st], ((t / kNst) - 1) & 1, abort_flag, a.status)))
                    break;
                uint8_t* dst = base + st * KV_BYTES;
                int lj;
                const int cons = tile_cons(t, n_pt, nla, nlb, has_b, &lj);
                if (lj < 0) {
                    one([&] { mbar_arrive_expect_tx(&full[st], KV_BYTES); });
                    tma_load_groups16_warp<NH>(dst, kHalf, mp, mp64, grp_row, t * 16, G, &full[st]);
                } else {
                    one([&] { mbar_arrive_expect_tx(&full[st], 2 * NH * box_bytes); });
                    const int X = cons == 2 ? 1 : 0;
                    const int U = X ? UB : UA;
                    for (int hb = 0; hb < 2; ++hb) {
                        const int L = uni_blk[X * ucap + min(2 * lj + hb, U - 1)];
                        const BlockBox kbb = block_box(g, L % g.nbf);
                        // first ring frame of the block's group (groups never wrap the ring)
                        const int cf = b * g.W + (a.ring_head + (L / g.nbf) * g.bt) % g.W;
                        for (int hh = 0; hh < NH; ++hh)
                            one([&] {
                                tma_load_5d(dst + hh * kHalf + hb * (kHalf / 2), ml, &full[st], hh * 64, h,
                                            kbb.x0, kbb.y0, cf);
                            });
                    }
                }
                ++issued;
            }
            if (lane == 0 && *abort_flag) {
                // let the copies already issued land before the CTA leaves
                if (isK) mbar_wait_drain(&bars[B_Q], 0, 100000000ull);
                for (int t = max(0, issued - kNst); t < issued; ++t)
                    mbar_wait_drain(&full[t % kNst], (t / kNst) & 1, 100000000ull);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------- MMA issuer
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
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
            bool ok = wwait(&bars[B_Q], 0);
            // per-side state, indexed only by the unrolled side loops (so it stays in registers)
            int pend[2] = {-1, -1};    // stream tile whose PV is still to be issued, per side
            int nqk[2] = {0, 0};       // QK MMAs issued per side
            int npv[2] = {0, 0};       // PV MMAs issued per side
            static_assert(kNst == 2, "two V stages");
            int vrem0 = 0, vrem1 = 0;  // PVs still to read each V stage
            const int n_side[2] = {n_side0, n_side1};
            auto issue_pv = [&](int X) -> bool {
                const int t = pend[X], st = t % kNst;
                if (!wwait(&bars[B_PF + X], npv[X] & 1)) return false;
                if (!wwait(&bars[B_VF + st], (t / kNst) & 1)) return false;
                tc_fence_after();
                const uint32_t p_tmem = tmem + 128 * X;
                const uint32_t o_tmem = tmem + 256 + 128 * X;
                const uint32_t v_base = smem_u32(sV + st * KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(o_tmem, p_tmem + kk * 8, sdesc_make(sdesc_lo(v_base, kHalf) + kk * 128), idesc_pv,
                            (npv[X] > 0 || kk > 0) ? 1u : 0u);
                commit(&bars[B_PV + X]);
                ++npv[X];
                const int left = st ? --vrem1 : --vrem0;
                if (left == 0) commit(&bars[B_VE + st]);
                pend[X] = -1;
                return true;
            };
            for (int t = 0; ok && t < n_stream; ++t) {
                const int st = t % kNst;
                if (!wwait(&bars[B_KF + st], (t / kNst) & 1)) { ok = false; break; }
                int lj;
                const int cons = tile_cons(t, n_pt, nla, nlb, has_b, &lj);
                const uint32_t k_base = smem_u32(sK + st * KV_BYTES);
#pragma unroll
                for (int X = 0; X < 2; ++X) {
                    if (cons & (1 << X)) {
                        if (pend[X] >= 0 && !issue_pv(X)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t q_base = smem_u32(sQ + X * Q_SIDE);
                        const uint32_t s_tmem = tmem + 128 * X;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                            mma_ss(s_tmem, sdesc_make(sdesc_lo(q_base, 16) + (off >> 4)), sdesc_make(sdesc_lo(k_base, 16) + (off >> 4)),
                                    idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        commit(&bars[B_SF + X]);
                        ++nqk[X];
                        pend[X] = t;
                    } else if (pend[X] >= 0 && nqk[X] == n_side[X]) {
                        // this side has no more tiles: finish it now so its V stage frees up
                        if (!issue_pv(X)) { ok = false; break; }
                    }
                }
                if (!ok) break;
                commit(&bars[B_KE + st]);
                if (st) vrem1 = __popc(cons);
                else vrem0 = __popc(cons);
            }
#pragma unroll
            for (int X = 0; X < 2; ++X)
                if (ok && pend[X] >= 0 && !issue_pv(X)) ok = false;
            if (!ok) {
                // wait for the MMAs already issued before TMEM is released
                commit(&bars[B_DRAIN]);
                mbar_wait_drain(&bars[B_DRAIN], 0, 100000000ull);
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ------------------------------------------------------ softmax warpgroups
        const int X = warp >> 2;          // side
        const int r = threadIdx.x & 127;  // query row of the side's tile = TMEM lane
        const int wq = warp & 3;          // lane quarter
        const int nX = X ? n_side1 : n_side0;
        const int hq = r >> 6;
        // token of this row in the chunk, or -1 for a padding row (computed in the epilogue,
        // where it is needed, so that nothing of it stays live in the loop)
        auto row_token = [&]() -> long long {
            const int qbr = qblock(X, hq);
            if (qbr < 0) return -1;
            const BlockBox qbb = block_box(g, qbr % g.nbf);
            int qt, qy, qx;
            if (!block_row(g, qbb, r & 63, &qt, &qy, &qx)) return -1;
            return (long long)((qbr / g.nbf) * g.bt + qt) * g.tf + (qbb.y0 + qy) * g.fw + qbb.x0 + qx;
        };
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t s_col = 128 * X, o_col = 256 + 128 * X;
        const float sl2 = kLog2e / sqrtf(static_cast<float>(D));
        const int U = X ? UB : UA;
        const int32_t* ublk = uni_blk + X * ucap;
        const int32_t* ubits = uni_bits + X * ucap;
        const size_t scratch_base =
            (((size_t)(bh * ka.n_groups + grp) * 2 + X) * a.n_seg_max) * 128 + r;
        float m = -CUDART_INF_F, l = 0.f, carry = 0.f;
        bool ok = true;
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.status));
        };
        auto emit = [&](int seg, float v, float mu) {
            if (MASS) a.scratch[scratch_base + (size_t)seg * 128] = v > 0.f ? mu + fast_log2(v) : -CUDART_INF_F;
        };

        for (int k = 0; k < nX; ++k) {
            if (!wwait(&bars[B_SF + X], k & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t s_addr = tmem + lane_base + s_col;
            float x[128];
            auto load_s = [&]() {
                uint32_t v[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + 32 * c, v[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[32 * c + e] = __uint_as_float(v[c][e]);
            };
            const bool persistent = k < n_pt;
            const int lj = persistent ? 0 : k - n_pt;
            // valid-column masks of the tile (64 bits per half); recomputed where they are
            // applied so that only the `masked` flag stays live across the exponentials
            auto tile_masks = [&](uint64_t& m0, uint64_t& m1) {
                if (persistent) {
                    const uint4 tm = tile_mask[k];
                    m0 = (static_cast<uint64_t>(tm.y) << 32) | tm.x;
                    m1 = (static_cast<uint64_t>(tm.w) << 32) | tm.z;
                } else {
                    const int u0 = 2 * lj;
                    const bool has1 = u0 + 1 < U;
                    const int L0 = ublk[u0], L1 = has1 ? ublk[u0 + 1] : L0;
                    const bool sel0 = (ubits[u0] >> hq) & 1;
                    const bool sel1 = has1 && ((ubits[u0 + 1] >> hq) & 1);
                    m0 = sel0 ? blk_mask[L0 % g.nbf] : 0ull;
                    m1 = sel1 ? blk_mask[L1 % g.nbf] : 0ull;
                }
            };
            bool masked;
            {
                uint64_t m0, m1;
                tile_masks(m0, m1);
                masked = (m0 & m1) != ~0ull;
            }
            auto apply_mask = [&]() {
                uint64_t mk0, mk1;
                tile_masks(mk0, mk1);
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    if (!((mk0 >> c) & 1ull)) x[c] = -CUDART_INF_F;
                    if (!((mk1 >> c) & 1ull)) x[64 + c] = -CUDART_INF_F;
                }
            };
            // Optimistic pass: the first half's exponentials against the running reference m
            // (what the lazy rescale uses whenever no row's maximum grew by more than 2^8),
            // with the tile's row maximum taken in the same pass.  Only when some row of the
            // warp needs a new reference (and always on the first tile) does the warp rescale
            // O and l and run the pass once more from S (still intact in TMEM: nothing is
            // stored yet); the second pass never needs a new reference, and the loop keeps one
            // copy of the pass in the code.
            float gs[16];
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                load_s();
                if (masked) apply_mask();
                const float mu0 = (m == -CUDART_INF_F) ? 0.f : m;
                const float mt = exp_half0_max(x, sl2, mu0, gs);
                const float m_new = fmaxf(m, mt * sl2);
                const bool need = m_new > m + 8.0f;
                if (!__any_sync(0xffffffffu, need)) break;
                const float alpha = need ? fast_exp2(m - m_new) : 1.0f;
                if (k > 0) {
                    if (!wwait(&bars[B_PV + X], (k - 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t v[32];
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        const uint32_t o_addr = tmem + lane_base + o_col + 32 * c;
                        tmem_ld32(o_addr, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                        tmem_st32(o_addr, v);
                    }
                    tmem_st_wait();
                }
                if (need) {
                    l *= alpha;
                    carry *= alpha;
                    m = m_new;
                }
            }
            if (!ok) break;
            const float mu = (m == -CUDART_INF_F) ? 0.f : m;
            // each half's P (bf16) goes over the first 64 columns of S as soon as it is done, so
            // the first store overlaps the second half's exponentials
            {
                uint32_t v0[32], v1[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) v0[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
                tmem_st32(s_addr, v0);
                exp_half<1>(x, sl2, mu, gs);
#pragma unroll
                for (int e = 0; e < 32; ++e) v1[e] = pack_bf16x2(x[64 + 2 * e], x[64 + 2 * e + 1]);
                tmem_st32(s_addr + 32, v1);
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(&bars[B_PF + X]);
            // row sum and mass bookkeeping (off the MMA's critical path)
            float s8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) s8[j] = gs[2 * j] + gs[2 * j + 1];
            const float p0 = (s8[0] + s8[1]) + (s8[2] + s8[3]);
            const float p1 = (s8[4] + s8[5]) + (s8[6] + s8[7]);
            l += p0 + p1;
            if (MASS) {
                if (persistent) {
                    // slots are runs of groups; emit each slot's partial where its run ends
                    const uint32_t ends = tile_end[k];
                    int seg = tile_seg[k];
#pragma unroll
                    for (int gq = 0; gq < 16; ++gq) {
                        carry += gs[gq];
                        if ((ends >> gq) & 1u) {
                            emit(seg, carry, mu);
                            ++seg;
                            carry = 0.f;
                        }
                    }
                } else {
                    emit(n_occ + 2 * lj, p0, mu);
                    if (2 * lj + 1 < U) emit(n_occ + 2 * lj + 1, p1, mu);
                }
            }
        }

        // --------------------------------------------------------------- epilogue
        const int bar_id = 1 + X;
        ok = named_bar_and(bar_id, 128, ok);
        if (ok && nX > 0) {
            ok = named_bar_and(bar_id, 128, wwait(&bars[B_PV + X], (nX - 1) & 1));
            tc_fence_after();
        }
        if (ok && nX > 0) {
            uint8_t* sO = sQ + X * Q_SIDE;  // the side's Q tile is free once its MMAs are done
            const float inv_l = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + o_col + 32 * c, v);
                tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 pk;
                    pk.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * inv_l, __uint_as_float(v[8 * q4 + 1]) * inv_l);
                    pk.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv_l, __uint_as_float(v[8 * q4 + 3]) * inv_l);
                    pk.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv_l, __uint_as_float(v[8 * q4 + 5]) * inv_l);
                    pk.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv_l, __uint_as_float(v[8 * q4 + 7]) * inv_l);
                    const int chunk = 4 * c + q4;
                    *reinterpret_cast<uint4*>(sO + (chunk >> 3) * kHalf + sw128_offset(r, chunk & 7)) = pk;
                }
            }
            const float lse2 = (l > 0.f) ? m + fast_log2(l) : -CUDART_INF_F;
            const long long q_tok = row_token();
            const bool row_valid = q_tok >= 0;
            if (row_valid) a.lse[(size_t)bh * a.q_frames * g.tf + q_tok] = lse2 * 0.6931471805599453f;
            fence_proxy_async_smem();
            named_bar_sync(bar_id, 128);
            if (r == 0) {
                for (int hb = 0; hb < 2; ++hb) {
                    const int qb = qblock(X, hb);
                    if (qb < 0) break;
                    const BlockBox obb = block_box(g, qb % g.nbf);
                    const int f0 = b * a.q_frames + (qb / g.nbf) * g.bt;
                    for (int hh = 0; hh < NH; ++hh)
                        tma_store_5d(&a.tm_o, sO + hh * kHalf + hb * (kHalf / 2), hh * 64, h, obb.x0, obb.y0, f0);
                }
                tma_store_commit();
                tma_store_wait_all();
            }
            if (MASS) {
                // one thread per slot/block: sum its 128 row partials, each normalised by its
                // row's log-sum-exp (padding rows carry +inf and add nothing)
                float* ls = lse_s + X * 128;
                ls[r] = row_valid ? lse2 : CUDART_INF_F;
                named_bar_sync(bar_id, 128);
                const int n_seg = n_occ + U;
                const float* side_base = a.scratch + (scratch_base - r);
                for (int sg = r; sg < n_seg; sg += 128) {
                    const float4* src = reinterpret_cast<const float4*>(side_base + (size_t)sg * 128);
                    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
                    for (int q = 0; q < 32; ++q) {
                        const float4 v = src[q];
                        const float4 w = reinterpret_cast<const float4*>(ls)[q];
                        acc0 += fast_exp2(v.x - w.x) + fast_exp2(v.y - w.y);
                        acc1 += fast_exp2(v.z - w.z) + fast_exp2(v.w - w.w);
                    }
                    const float v = acc0 + acc1;
                    if (sg < n_occ) {
                        if (a.mass_pers) atomicAdd(&a.mass_pers[(size_t)bh * S + seg_slot[sg]], v);
                    } else {
                        const int L = ublk[sg - n_occ];
                        const int phys = (head_g + L / g.nbf) % g.Wg;
                        if (a.mass_local)
                            atomicAdd(&a.mass_local[((size_t)bh * g.Wg + phys) * g.nbf + L % g.nbf], v);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 10) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmCols);
    }
}

template <int D, bool MASS>
cudaError_t launch_fwd_t(const FwdKernelArgs& ka, dim3 grid, size_t smem, cudaStream_t st) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, MASS>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;  // register split needs it
    e = cudaFuncSetAttribute(attn_fwd_kernel<D, MASS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_fwd_kernel<D, MASS><<<grid, kThreads, smem, st>>>(ka);
    return cudaGetLastError();
}

}  // namespace

size_t attn_fwd_smem_bytes(const Geo& g, int ucap) {
    // at least 120 KB so that one CTA (holding all 512 TMEM columns) runs per SM
    const size_t need = fwd_plan(g.D, g.S, ucap, g.nbf).total + 1024;
    return need < 120 * 1024 ? 120 * 1024 : need;
}

cudaError_t launch_attn_fwd(const FwdArgs& a, bool with_mass, cudaStream_t st) {
    FwdKernelArgs ka;
    ka.a = a;
    ka.n_groups = (a.q_frames / a.g.bt * a.g.nbf + 3) / 4;
    const size_t smem = attn_fwd_smem_bytes(a.g, a.ucap);
    dim3 grid(ka.n_groups, a.g.H, a.g.B);
    if (a.g.D == 128)
        return with_mass ? launch_fwd_t<128, true>(ka, grid, smem, st)
                         : launch_fwd_t<128, false>(ka, grid, smem, st);
    return with_mass ? launch_fwd_t<64, true>(ka, grid, smem, st)
                     : launch_fwd_t<64, false>(ka, grid, smem, st);
}

}  // namespace pbsa
