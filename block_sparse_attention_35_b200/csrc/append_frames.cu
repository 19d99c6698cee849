// append_frames.cu - frames joining the PBSA cache, fused with the key-mean cache.
//
// Each chunk's frames enter the KV cache (pith.science page, algorithm fragment: the KV
// pass of a chunk writes its keys and values).  Frames of the sequence's sink (project
// page, kernel features: the "sink" sparsity pattern) go, block by block, into their
// reserved persistent slots; every other frame goes into the local window's ring.  A
// window block never changes while it is cached, so its mean key (the block score's key
// side) is computed here, in the same pass that copies it, and kept by ring frame group
// for pbsa_select_blocks_pooled.
//
// append_kernel: one CTA per (block of the new frames, batch item).  Each thread owns 8
// consecutive channels of a token's [H, D] row (a CTA moves whole 3 KB rows of all heads,
// fully coalesced), streams the block's valid tokens with 16-byte loads (up to eight rows of
// K and V in flight), stores K and V to their destination and, for window
// blocks, sums K for the mean in the order pool_kernel does (so the means are identical).
// HBM traffic per appended frame: its K and V read once and written once.
#include <cuda_bf16.h>

#include "pbsa_device.cuh"
#include "pbsa_internal.cuh"

namespace pbsa {

namespace {

struct AppendParams {
    Geo g;
    const __nv_bfloat16* ks;  // [B, n_frames * T_f, H, D]
    const __nv_bfloat16* vs;
    int n_frames;             // frames of the source
    int n_sink;               // its first n_sink frames are sink frames
    int sink_group0;          // global frame group of the first source frame
    int ring_slot;            // ring frame of the first window frame of the source
    __nv_bfloat16* kl;        // ring [B, W * T_f, H, D]
    __nv_bfloat16* vl;
    float* kbar;              // nullable, [B, H, Wg * NB, D]
    __nv_bfloat16* kp;        // [B, H, S, 64, D]
    __nv_bfloat16* vp;
    int32_t* pers_len;
    float* pers_score;
    int32_t* pers_src;
};

// ROWS token rows in flight per thread: 8 when the CTA has at most 512 threads
// (H*D <= 4096), else 4 so that 1024 threads fit in the register file.
template <int ROWS>
__global__ void __launch_bounds__(ROWS > 4 ? 512 : 1024) append_kernel(AppendParams p) {
    const Geo& g = p.g;
    const int j = blockIdx.x, b = blockIdx.y;
    const int hd = g.H * g.D;
    const int t8 = threadIdx.x * 8;
    const int grp = j / g.nbf, i = j % g.nbf;       // frame group of the source, block
    const int f0 = grp * g.bt;                       // its first source frame
    const bool sink = f0 < p.n_sink;
    const BlockBox bb = block_box(g, i);
    const int plane = bb.hv * bb.wv, n = g.bt * plane;
    const int h = t8 / g.D, d0 = t8 % g.D;
    const int slot = (p.sink_group0 + grp) * g.nbf + i;               // sink destination
    const int ring_f0 = (p.ring_slot + f0 - p.n_sink) % g.W;          // window destination
    if (sink && threadIdx.x < g.H) {
        const size_t m = ((size_t)b * g.H + threadIdx.x) * g.S + slot;
        p.pers_len[m] = n;
        p.pers_score[m] = 0.f;
        p.pers_src[m] = slot;
    }
    if (t8 >= hd) return;

    const __nv_bfloat16* ksrc = p.ks + ((long long)b * p.n_frames + f0) * g.tf * hd + t8;
    const __nv_bfloat16* vsrc = p.vs + ((long long)b * p.n_frames + f0) * g.tf * hd + t8;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    constexpr int kRows = ROWS;
    for (int r0 = 0; r0 < n; r0 += kRows) {
        uint4 kv[kRows], vv[kRows];
        long long off[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const int r = r0 + u;
            if (r < n) {
                const int t = r / plane, y = bb.y0 + (r % plane) / bb.wv, x = bb.x0 + r % bb.wv;
                off[u] = (long long)t * g.tf + y * g.fw + x;   // token offset from the group's first frame
                kv[u] = __ldg(reinterpret_cast<const uint4*>(ksrc + off[u] * hd));
                vv[u] = __ldg(reinterpret_cast<const uint4*>(vsrc + off[u] * hd));
            }
        }
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const int r = r0 + u;
            if (r >= n) continue;
            if (sink) {
                const size_t dst = ((((size_t)b * g.H + h) * g.S + slot) * 64 + r) * g.D + d0;
                *reinterpret_cast<uint4*>(p.kp + dst) = kv[u];
                *reinterpret_cast<uint4*>(p.vp + dst) = vv[u];
            } else {
                const size_t dst = (((size_t)b * g.W + ring_f0) * g.tf + off[u]) * hd + t8;
                *reinterpret_cast<uint4*>(p.kl + dst) = kv[u];
                *reinterpret_cast<uint4*>(p.vl + dst) = vv[u];
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&kv[u]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h2[e]);
                    acc[2 * e] += f.x;
                    acc[2 * e + 1] += f.y;
                }
            }
        }
    }
    if (sink) {
        // rows past the block's length: zero (the attention kernels need them finite)
        for (int r = n; r < 64; ++r) {
            const size_t dst = ((((size_t)b * g.H + h) * g.S + slot) * 64 + r) * g.D + d0;
            *reinterpret_cast<uint4*>(p.kp + dst) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(p.vp + dst) = make_uint4(0, 0, 0, 0);
        }
    } else if (p.kbar) {
        const int row = (ring_f0 / g.bt) * g.nbf + i;
        float* out = p.kbar + (((size_t)b * g.H + h) * g.Wg * g.nbf + row) * g.D + d0;
        const float c = static_cast<float>(n);
        reinterpret_cast<float4*>(out)[0] = make_float4(acc[0] / c, acc[1] / c, acc[2] / c, acc[3] / c);
        reinterpret_cast<float4*>(out)[1] = make_float4(acc[4] / c, acc[5] / c, acc[6] / c, acc[7] / c);
    }
}

}  // namespace

cudaError_t launch_append(const Geo& g, const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                          int n_frames, int n_sink, int sink_group0, __nv_bfloat16* k_local,
                          __nv_bfloat16* v_local, int ring_slot, float* kbar, __nv_bfloat16* k_pers,
                          __nv_bfloat16* v_pers, int32_t* pers_len, float* pers_score,
                          int32_t* pers_src, cudaStream_t st) {
    const int nblk = n_frames / g.bt * g.nbf;
    if (nblk == 0) return cudaSuccess;
    AppendParams p{g, k_new, v_new, n_frames, n_sink, sink_group0, ring_slot, k_local, v_local, kbar,
                   k_pers, v_pers, pers_len, pers_score, pers_src};
    const int threads = (g.H * g.D / 8 + 31) / 32 * 32;
    if (threads <= 512)
        append_kernel<8><<<dim3(nblk, g.B), threads, 0, st>>>(p);
    else
        append_kernel<4><<<dim3(nblk, g.B), threads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace pbsa
