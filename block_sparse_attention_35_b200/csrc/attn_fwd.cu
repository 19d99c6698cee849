// attn_fwd.cu - PBSA forward on sm_100a (TMA + tcgen05 + TMEM).
//
// Sparse Forcing (pith.science abstract; project page kernel features): every query token
// attends to all blocks of the persistent cache and to the top-k blocks of the local
// window selected for its query block, with softmax scale 1/sqrt(D).  With a mass output
// the kernel also accumulates, per persistent slot and per local block, the softmax
// probability summed over the chunk's query rows (the score that ranks blocks when the
// window slides).
//
// One CTA = one 128-row query tile = two 8x8 query blocks of one (batch, head), each
// loaded as a 64-row 5-D TMA box [1 frame, 8 rows, 8 cols, 1 head, 64 channels]; rows of
// ragged edge blocks fall outside the tensor and are zero-filled on load and clipped on
// store.  Key tiles are 128 keys:
//   * persistent phase: the occupied slots' valid rows, compacted into a stream of 8-row
//     groups (slot lengths are multiples of 8), 16 groups per tile, each group one 2-D TMA
//     box; only the last tile is partial;
//   * local phase: the union of the two query blocks' selections, two 8x8 key blocks per
//     tile, each a 5-D TMA box from the ring; columns of a block the row's query block did
//     not select, or outside the frame, are masked.
// Warp roles (192 threads): warps 0-3 softmax (one query row per thread), warp 4 TMA
// producer, warp 5 MMA issuer.  TMEM: S double buffer (2 x 128 columns) and the O
// accumulator (D columns).  S = Q K^T is an SS MMA (both operands K-major, 128-byte
// swizzle); P is converted to bf16 in registers and written back over S in TMEM, and
// O += P V is a TS MMA (A from TMEM, V MN-major in shared memory).  O is rescaled only
// when a row maximum grows by more than 2^8 (exponentials stay <= 256).
// Mass: while streaming, each row emits for every slot/block it saw the log2 of its
// partial probability sum (relative to the running maximum) into per-CTA scratch; after
// the final log-sum-exp is known the CTA turns them into probabilities, sums over rows
// and adds one value per slot/block to the global mass arrays.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

constexpr int kNst = 2;               // K/V pipeline stages
constexpr uint32_t kHalf = 128 * 128; // bytes of 128 rows x 64 bf16 channels
constexpr uint32_t kTmS0 = 0, kTmS1 = 128, kTmO = 256, kTmCols = 512;
constexpr int kThreads = 192;

struct SmemPlan {
    uint32_t q, k, v, grp_row, grp_seg, seg_slot, uni_blk, uni_bits, seg_mass, bars, misc,
        total;
};

__host__ __device__ inline SmemPlan fwd_plan(int D, int S, int ucap) {
    SmemPlan p;
    const uint32_t nh = D / 64;
    p.q = 0;
    p.k = p.q + nh * kHalf;
    p.v = p.k + kNst * nh * kHalf;
    p.grp_row = p.v + kNst * nh * kHalf;
    p.grp_seg = p.grp_row + 4u * 8u * S;
    p.seg_slot = p.grp_seg + 4u * 8u * S;
    p.uni_blk = p.seg_slot + 4u * S;
    p.uni_bits = p.uni_blk + 4u * ucap;
    p.seg_mass = p.uni_bits + 4u * ucap;
    p.bars = (p.seg_mass + 4u * (S + ucap) + 7u) & ~7u;
    p.misc = p.bars + 8u * 16u;
    p.total = p.misc + 4u * 8u;
    return p;
}

// barrier slots
enum { B_Q = 0, B_KF = 1, B_VF = 3, B_KE = 5, B_SF = 7, B_PF = 9, B_PV = 11, B_DRAIN = 13 };
// misc slots
enum { M_TMEM = 0, M_ABORT = 1, M_G = 2, M_OCC = 3, M_U = 4 };

struct FwdKernelArgs {
    FwdArgs a;
    int ucap;
    int n_ctiles;  // query tiles per (b, h)
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int D, bool MASS>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdKernelArgs ka) {
    constexpr int NH = D / 64;
    constexpr uint32_t KV_BYTES = NH * kHalf;
    const FwdArgs& a = ka.a;
    const Geo& g = a.g;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int S = g.S;
    const int ucap = ka.ucap;
    const SmemPlan P = fwd_plan(D, S, ucap);
    uint8_t* sQ = sm + P.q;
    uint8_t* sK = sm + P.k;
    uint8_t* sV = sm + P.v;
    int32_t* grp_row = reinterpret_cast<int32_t*>(sm + P.grp_row);
    int32_t* grp_seg = reinterpret_cast<int32_t*>(sm + P.grp_seg);
    int32_t* seg_slot = reinterpret_cast<int32_t*>(sm + P.seg_slot);
    int32_t* uni_blk = reinterpret_cast<int32_t*>(sm + P.uni_blk);
    int32_t* uni_bits = reinterpret_cast<int32_t*>(sm + P.uni_bits);
    float* seg_mass = reinterpret_cast<float*>(sm + P.seg_mass);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P.bars);
    int* misc = reinterpret_cast<int*>(sm + P.misc);
    volatile int* abort_flag = misc + M_ABORT;

    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * g.H + h;
    const int qb_total = a.q_frames * g.nbf;
    const int qb0 = 2 * tile;
    const int qb1 = (2 * tile + 1 < qb_total) ? 2 * tile + 1 : -1;
    const int nl = a.local_frames * g.nbf;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ------------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        mbar_init(&bars[B_Q], 1);
        for (int s = 0; s < kNst; ++s) {
            mbar_init(&bars[B_KF + s], 1);
            mbar_init(&bars[B_VF + s], 1);
            mbar_init(&bars[B_KE + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[B_SF + s], 1);
            mbar_init(&bars[B_PF + s], 128);
            mbar_init(&bars[B_PV + s], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        misc[M_ABORT] = 0;
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(reinterpret_cast<uint32_t*>(misc + M_TMEM), kTmCols);
    if (warp == 0) {
        // compacted stream of the occupied slots' 8-row groups
        int run = 0, occ = 0;
        for (int s0 = 0; s0 < S; s0 += 32) {
            const int s = s0 + lane;
            int len = (s < S) ? a.pers_len[(size_t)bh * S + s] : 0;
            if (len < 0 || len > 64 || (len & 7)) {
                set_status(a.status, PBSA_ERR_DEVICE_CHECK);
                len = 0;
            }
            const int ng = len >> 3, oc = ng > 0 ? 1 : 0;
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
                    grp_row[gstart + i] = ((bh * S) + s) * 64 + 8 * i;
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
    }
    if (warp == 1 && lane == 0) {
        // union of the two query blocks' selections (both lists ascending)
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
        misc[M_U] = u;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = static_cast<uint32_t>(misc[M_TMEM]);
    const int G = misc[M_G], n_occ = misc[M_OCC], U = misc[M_U];
    const int n_pt = (G + 15) / 16;
    const int n_tiles = n_pt + (U + 1) / 2;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&a.tm_q);
            tma_prefetch_desc(&a.tm_kp);
            tma_prefetch_desc(&a.tm_vp);
            tma_prefetch_desc(&a.tm_kl);
            tma_prefetch_desc(&a.tm_vl);
            mbar_arrive_expect_tx(&bars[B_Q], 2 * NH * (kHalf / 2));
            for (int hb = 0; hb < 2; ++hb) {
                const int qb = (hb == 1 && qb1 >= 0) ? qb1 : qb0;
                const int f = qb / g.nbf, i = qb % g.nbf;
                const int by = i / g.nbx, bx = i % g.nbx;
                for (int hh = 0; hh < NH; ++hh)
                    tma_load_5d(sQ + hh * kHalf + hb * (kHalf / 2), &a.tm_q, &bars[B_Q], hh * 64, h,
                                8 * bx, 8 * by, b * a.q_frames + f);
            }
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int st = it % kNst;
                if (it >= kNst &&
                    !mbar_wait(&bars[B_KE + st], ((it / kNst) - 1) & 1, abort_flag, a.status))
                    break;
                uint8_t* dk = sK + st * KV_BYTES;
                uint8_t* dv = sV + st * KV_BYTES;
                mbar_arrive_expect_tx(&bars[B_KF + st], KV_BYTES);
                if (it < n_pt) {
                    for (int c = 0; c < 16; ++c) {
                        const int row = grp_row[min(it * 16 + c, G - 1)];
                        for (int hh = 0; hh < NH; ++hh)
                            tma_load_2d(dk + hh * kHalf + c * 1024, &a.tm_kp, &bars[B_KF + st],
                                        hh * 64, row);
                    }
                    mbar_arrive_expect_tx(&bars[B_VF + st], KV_BYTES);
                    for (int c = 0; c < 16; ++c) {
                        const int row = grp_row[min(it * 16 + c, G - 1)];
                        for (int hh = 0; hh < NH; ++hh)
                            tma_load_2d(dv + hh * kHalf + c * 1024, &a.tm_vp, &bars[B_VF + st],
                                        hh * 64, row);
                    }
                } else {
                    const int j = it - n_pt;
                    int crd[2][3];
                    for (int hb = 0; hb < 2; ++hb) {
                        const int L = uni_blk[min(2 * j + hb, U - 1)];
                        const int pos = L / g.nbf, i = L % g.nbf;
                        crd[hb][0] = 8 * (i % g.nbx);
                        crd[hb][1] = 8 * (i / g.nbx);
                        crd[hb][2] = b * g.W + (a.ring_head + pos) % g.W;
                    }
                    for (int hb = 0; hb < 2; ++hb)
                        for (int hh = 0; hh < NH; ++hh)
                            tma_load_5d(dk + hh * kHalf + hb * (kHalf / 2), &a.tm_kl,
                                        &bars[B_KF + st], hh * 64, h, crd[hb][0], crd[hb][1],
                                        crd[hb][2]);
                    mbar_arrive_expect_tx(&bars[B_VF + st], KV_BYTES);
                    for (int hb = 0; hb < 2; ++hb)
                        for (int hh = 0; hh < NH; ++hh)
                            tma_load_5d(dv + hh * kHalf + hb * (kHalf / 2), &a.tm_vl,
                                        &bars[B_VF + st], hh * 64, h, crd[hb][0], crd[hb][1],
                                        crd[hb][2]);
                }
                ++issued;
            }
            if (*abort_flag) {
                // let the copies already issued land before the CTA leaves
                mbar_wait_drain(&bars[B_Q], 0, 100000000ull);
                for (int it = max(0, issued - kNst); it < issued; ++it) {
                    const int st = it % kNst;
                    mbar_wait_drain(&bars[B_KF + st], (it / kNst) & 1, 100000000ull);
                    mbar_wait_drain(&bars[B_VF + st], (it / kNst) & 1, 100000000ull);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
            const uint32_t q_base = smem_u32(sQ);
            bool ok = mbar_wait(&bars[B_Q], 0, abort_flag, a.status);
            auto issue_pv = [&](int j) -> bool {
                const int sbj = j & 1, stj = j % kNst;
                if (!mbar_wait(&bars[B_PF + sbj], (j >> 1) & 1, abort_flag, a.status)) return false;
                if (!mbar_wait(&bars[B_VF + stj], (j / kNst) & 1, abort_flag, a.status)) return false;
                tc_fence_after();
                const uint32_t p_tmem = tmem + (sbj ? kTmS1 : kTmS0);
                const uint32_t v_base = smem_u32(sV + stj * KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bdesc = sdesc_sw128(v_base + kk * 2048, kHalf, 1024);
                    umma_ts(tmem + kTmO, p_tmem + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[B_PV + sbj]);
                umma_commit(&bars[B_KE + stj]);
                return true;
            };
            for (int it = 0; ok && it < n_tiles; ++it) {
                const int st = it % kNst, sb = it & 1;
                if (!mbar_wait(&bars[B_KF + st], (it / kNst) & 1, abort_flag, a.status)) { ok = false; break; }
                if (it >= 2 && !mbar_wait(&bars[B_PV + sb], ((it - 2) >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t s_tmem = tmem + (sb ? kTmS1 : kTmS0);
                const uint32_t k_base = smem_u32(sK + st * KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                    const uint64_t adesc = sdesc_sw128(q_base + off, 16, 1024);
                    const uint64_t bdesc = sdesc_sw128(k_base + off, 16, 1024);
                    umma_ss(s_tmem, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars[B_SF + sb]);
                if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
            }
            if (ok && n_tiles > 0) ok = issue_pv(n_tiles - 1);
            if (!ok) {
                // wait for the MMAs already issued before TMEM is released
                umma_commit(&bars[B_DRAIN]);
                mbar_wait_drain(&bars[B_DRAIN], 0, 100000000ull);
            }
        }
    } else {
        // --------------------------------------------------------- softmax warps
        const int r = threadIdx.x;  // query row of the tile = TMEM lane
        const int hq = r >> 6, rr = r & 63, dy = rr >> 3, dx = rr & 7;
        const int qbr = hq ? qb1 : qb0;
        const int qbv = qbr >= 0 ? qbr : qb0;
        const int qf = qbv / g.nbf, qi = qbv % g.nbf;
        const int qy = 8 * (qi / g.nbx) + dy, qx = 8 * (qi % g.nbx) + dx;
        const bool row_valid = qbr >= 0 && qy < g.fh && qx < g.fw;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
        const size_t scratch_base =
            ((size_t)(bh * ka.n_ctiles + tile) * a.n_seg_max) * 128 + r;
        float m = -CUDART_INF_F, l = 0.f, carry = 0.f;
        int cur_seg = -1;
        bool ok = true;
        // every wait result is made warp-uniform: tcgen05.ld/st are warp-collective
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.status));
        };
        auto emit = [&](int seg, float v, float mu) {
            if (MASS) a.scratch[scratch_base + (size_t)seg * 128] = v > 0.f ? mu + fast_log2(v) : -CUDART_INF_F;
        };

        for (int it = 0; it < n_tiles; ++it) {
            const int sb = it & 1;
            if (!wwait(&bars[B_SF + sb], (it >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t s_addr = tmem + lane_base + (sb ? kTmS1 : kTmS0);
            float x[128];
            {
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld32(s_addr + 32 * c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[32 * c + e] = __uint_as_float(v[e]);
                }
            }
            // masks -> x in log2 units, -inf where masked
            if (it < n_pt) {
                const int nvc = min(128, 8 * (G - 16 * it));
#pragma unroll
                for (int c = 0; c < 128; ++c) x[c] = (c < nvc) ? x[c] * sl2 : -CUDART_INF_F;
            } else {
                const int j = it - n_pt;
                const int u0 = 2 * j;
                const bool has1 = u0 + 1 < U;
                const int L0 = uni_blk[u0], L1 = has1 ? uni_blk[u0 + 1] : L0;
                const bool sel0 = (uni_bits[u0] >> hq) & 1;
                const bool sel1 = has1 && ((uni_bits[u0 + 1] >> hq) & 1);
                const int i0 = L0 % g.nbf, i1 = L1 % g.nbf;
                const int hv0 = sel0 ? min(8, g.fh - 8 * (i0 / g.nbx)) : 0;
                const int wv0 = min(8, g.fw - 8 * (i0 % g.nbx));
                const int hv1 = sel1 ? min(8, g.fh - 8 * (i1 / g.nbx)) : 0;
                const int wv1 = min(8, g.fw - 8 * (i1 % g.nbx));
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    x[c] = ((c >> 3) < hv0 && (c & 7) < wv0) ? x[c] * sl2 : -CUDART_INF_F;
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    x[64 + c] = ((c >> 3) < hv1 && (c & 7) < wv1) ? x[64 + c] * sl2 : -CUDART_INF_F;
            }
            float mt = x[0];
#pragma unroll
            for (int c = 1; c < 128; ++c) mt = fmaxf(mt, x[c]);
            const float m_new = fmaxf(m, mt);
            const bool need = m_new > m + 8.0f;
            if (__any_sync(0xffffffffu, need)) {
                const float alpha = need ? fast_exp2(m - m_new) : 1.0f;
                if (it > 0) {
                    if (!wwait(&bars[B_PV + ((it - 1) & 1)], ((it - 1) >> 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t v[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        const uint32_t o_addr = tmem + lane_base + kTmO + 32 * c;
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
            const float mu = (m == -CUDART_INF_F) ? 0.f : m;
#pragma unroll
            for (int c = 0; c < 128; ++c) x[c] = fast_exp2(x[c] - mu);
            if (it < n_pt) {
#pragma unroll
                for (int gq = 0; gq < 16; ++gq) {
                    float gs = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) gs += x[8 * gq + e];
                    l += gs;
                    if (MASS) {
                        const int gi = 16 * it + gq;
                        if (gi < G) {
                            const int seg = grp_seg[gi];
                            if (seg != cur_seg) {
                                if (cur_seg >= 0) emit(cur_seg, carry, mu);
                                cur_seg = seg;
                                carry = 0.f;
                            }
                            carry += gs;
                        }
                    }
                }
                if (MASS && it == n_pt - 1 && cur_seg >= 0) {
                    emit(cur_seg, carry, mu);
                    cur_seg = -1;
                    carry = 0.f;
                }
            } else {
                float p0 = 0.f, p1 = 0.f;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    p0 += x[c];
                    p1 += x[64 + c];
                }
                l += p0 + p1;
                if (MASS) {
                    const int u0 = 2 * (it - n_pt);
                    emit(n_occ + u0, p0, mu);
                    if (u0 + 1 < U) emit(n_occ + u0 + 1, p1, mu);
                }
            }
            // P (bf16) over the first 64 columns of this S buffer
            {
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = pack_bf16x2(x[64 * c + 2 * e], x[64 * c + 2 * e + 1]);
                    tmem_st32(s_addr + 32 * c, v);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(&bars[B_PF + sb]);
        }

        // --------------------------------------------------------------- epilogue
        // one decision for all 128 softmax threads (the epilogue has named barriers)
        ok = named_bar_and(1, 128, ok);
        if (ok && n_tiles > 0) {
            const int jl = n_tiles - 1;
            ok = named_bar_and(1, 128, wwait(&bars[B_PV + (jl & 1)], (jl >> 1) & 1));
            tc_fence_after();
        }
        if (ok) {
            const float inv_l = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                if (n_tiles > 0) {
                    tmem_ld32(tmem + lane_base + kTmO + 32 * c, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 pk;
                    pk.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * inv_l, __uint_as_float(v[8 * q4 + 1]) * inv_l);
                    pk.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv_l, __uint_as_float(v[8 * q4 + 3]) * inv_l);
                    pk.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv_l, __uint_as_float(v[8 * q4 + 5]) * inv_l);
                    pk.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv_l, __uint_as_float(v[8 * q4 + 7]) * inv_l);
                    const int chunk = 4 * c + q4;  // 16-byte chunk of the row (8 channels)
                    const int hh = chunk >> 3;
                    *reinterpret_cast<uint4*>(sQ + hh * kHalf + sw128_offset(r, chunk & 7)) = pk;
                }
            }
            const float lse2 = (l > 0.f) ? m + fast_log2(l) : -CUDART_INF_F;
            if (row_valid)
                a.lse[(size_t)bh * a.q_frames * g.tf + qf * g.tf + qy * g.fw + qx] = lse2 * 0.6931471805599453f;
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (r == 0) {
                for (int hb = 0; hb < 2; ++hb) {
                    if (hb == 1 && qb1 < 0) break;
                    const int qb = hb ? qb1 : qb0;
                    const int f = qb / g.nbf, i = qb % g.nbf;
                    for (int hh = 0; hh < NH; ++hh)
                        tma_store_5d(&a.tm_o, sQ + hh * kHalf + hb * (kHalf / 2), hh * 64, h,
                                     8 * (i % g.nbx), 8 * (i / g.nbx), b * a.q_frames + f);
                }
                tma_store_commit();
                tma_store_wait_all();
            }
            if (MASS) {
                const int n_seg = n_occ + U;
                for (int s = r; s < n_seg; s += 128) seg_mass[s] = 0.f;
                named_bar_sync(1, 128);
                for (int s = 0; s < n_seg; ++s) {
                    float v = row_valid ? fast_exp2(a.scratch[scratch_base + (size_t)s * 128] - lse2) : 0.f;
                    v = warp_sum(v);
                    if (lane == 0) atomicAdd(&seg_mass[s], v);
                }
                named_bar_sync(1, 128);
                for (int s = r; s < n_seg; s += 128) {
                    const float v = seg_mass[s];
                    if (s < n_occ) {
                        if (a.mass_pers) atomicAdd(&a.mass_pers[(size_t)bh * S + seg_slot[s]], v);
                    } else {
                        const int L = uni_blk[s - n_occ];
                        const int phys = (a.ring_head + L / g.nbf) % g.W;
                        if (a.mass_local)
                            atomicAdd(&a.mass_local[((size_t)bh * g.W + phys) * g.nbf + L % g.nbf], v);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmCols);
    }
}

template <int D, bool MASS>
cudaError_t launch_fwd_t(const FwdKernelArgs& ka, dim3 grid, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, MASS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_fwd_kernel<D, MASS><<<grid, kThreads, smem, st>>>(ka);
    return cudaGetLastError();
}

}  // namespace

size_t attn_fwd_smem_bytes(const Geo& g, int ucap) {
    // at least 120 KB so that one CTA (holding all 512 TMEM columns) runs per SM
    const size_t need = fwd_plan(g.D, g.S, ucap).total + 1024;
    return need < 120 * 1024 ? 120 * 1024 : need;
}

cudaError_t launch_attn_fwd(const FwdArgs& a, bool with_mass, cudaStream_t st) {
    FwdKernelArgs ka;
    ka.a = a;
    ka.ucap = a.ucap;
    const int qb_total = a.q_frames * a.g.nbf;
    ka.n_ctiles = (qb_total + 1) / 2;
    const size_t smem = attn_fwd_smem_bytes(a.g, ka.ucap);
    dim3 grid(ka.n_ctiles, a.g.H, a.g.B);
    if (a.g.D == 128)
        return with_mass ? launch_fwd_t<128, true>(ka, grid, smem, st)
                         : launch_fwd_t<128, false>(ka, grid, smem, st);
    return with_mass ? launch_fwd_t<64, true>(ka, grid, smem, st)
                     : launch_fwd_t<64, false>(ka, grid, smem, st);
}

}  // namespace pbsa
