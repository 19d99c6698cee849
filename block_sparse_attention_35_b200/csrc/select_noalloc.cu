// select_noalloc.cu - block selection that allocates nothing and takes no workspace.
//
// Some callers cannot allocate device memory at the point where they need a block
// selection: a plugin inside an inference engine whose memory plan is fixed before it
// runs, or a decode loop that must never call cudaMalloc because it blocks the host and
// synchronises the device.  For them this file keeps the selection's scratch (the pooled
// query and key block means) in a library-owned static device array instead of a
// caller-provided workspace.  Every GPU that loads the library holds this array (8 MiB)
// until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "pbsa.h"
#include "pbsa_internal.cuh"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(PBSA_SELECT_STATIC_SCRATCH_BYTES);

// The scratch itself.  In host code this name is only a host-side stand-in for the
// device symbol, never a device address: the address is looked up below.
static __device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device, looked up once per device
// (with that device current) and cached.
int scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return pbsa::api_cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return pbsa::api_fail(PBSA_ERR_UNSUPPORTED, "device ordinal >= 64");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess) return pbsa::api_cuda_fail(e, "cudaGetSymbolAddress(select scratch)");
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return PBSA_OK;
}

}  // namespace

extern "C" PBSA_API int pbsa_select_blocks_noalloc(const pbsa_config* cfg, const void* q, int q_frames,
                                                   const void* k_local, int local_frames, int ring_head,
                                                   int32_t* idx, int idx_stride, int32_t* cnt,
                                                   float* scores, void* stream) {
    pbsa::Geo g;
    int k = 0;
    size_t need = 0, key_off = 0;
    int rc = pbsa::api_prepare_select(cfg, q, q_frames, k_local, local_frames, ring_head, idx, idx_stride,
                                      cnt, scores, &g, &k, &need, &key_off);
    if (rc != PBSA_OK) return rc;
    // every window block selected and no scores asked for: no scratch needed
    if (k == local_frames / g.bt * g.nbf && !scores) {
        cudaError_t e = pbsa::launch_select_all(g, q_frames / g.bt * g.nbf, k, idx, idx_stride, cnt,
                                                static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return pbsa::api_cuda_fail(e, "select-all kernel launch");
        return PBSA_OK;
    }
    if (need > kScratchBytes)
        return pbsa::api_fail(PBSA_ERR_UNSUPPORTED,
                              "selection needs more scratch than the 8 MiB static buffer of "
                              "pbsa_select_blocks_noalloc; call pbsa_select_blocks with a workspace");
    void* scratch = nullptr;
    if ((rc = scratch_address(&scratch)) != PBSA_OK) return rc;
    // Nothing in the scratch needs clearing: the pooling kernel writes every mean the
    // scoring kernel reads in the same call.
    float* qbar = static_cast<float*>(scratch);
    float* kbar = reinterpret_cast<float*>(static_cast<char*>(scratch) + key_off);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = pbsa::launch_pool(g, static_cast<const __nv_bfloat16*>(q), q_frames,
                                      static_cast<const __nv_bfloat16*>(k_local), ring_head, local_frames,
                                      qbar, kbar, st);
    if (e != cudaSuccess) return pbsa::api_cuda_fail(e, "pool kernel launch");
    e = pbsa::launch_score_topk(g, qbar, kbar, ring_head, q_frames / g.bt * g.nbf, local_frames / g.bt * g.nbf, k, idx, idx_stride,
                                cnt, scores, st);
    if (e != cudaSuccess) return pbsa::api_cuda_fail(e, "score/top-k kernel launch");
    return PBSA_OK;
}
