// Hierarchical volume decoding for callers that cannot allocate device memory.
//
// vdm_decode_hierarchical() takes its scratch space from the caller.  Some
// callers cannot provide it: code embedded in a host application that owns
// every byte of device memory (its own pool or a fixed budget) and does not
// let a library call cudaMalloc, and latency-critical callers that must not
// call cudaMalloc / cudaFree at all because those calls can synchronise the
// whole device.  vdm_decode_hierarchical_noalloc() serves them: its scratch is
// a fixed array compiled into this library, so neither the caller nor the
// library allocates anything.
//
// Costs and rules of that choice:
//   * every GPU that loads the library reserves kStaticScratchBytes (32 MiB)
//     for this array until the process exits;
//   * problems whose scratch need (vdm_hierarchical_workspace_size) is larger
//     than the array are rejected with VDM_ERR_UNSUPPORTED;
//   * all calls on a device share the one array, so calls that overlap on the
//     GPU (other streams, other host threads) race and corrupt each other's
//     results; serialise them on one stream.  The array keeps whatever the last
//     call left in it; the decoding writes every scratch word it later reads
//     and clears its counters itself, so stale contents do no harm;
//   * the first call on a device looks up the array's device address (a host
//     call that allocates nothing).
#include <mutex>

#include "vdm_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)32 << 20;
constexpr int kMaxDevices = 64;

// The scratch itself.  Host code must not use this name as a device address
// (on the host it is only a stand-in); it asks the runtime for the address.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

using namespace vdm;

extern "C" {

vdm_status vdm_decode_hierarchical_noalloc(const vdm_decoder* dec, const void* d_k, const void* d_v,
                                           int32_t B, int32_t N, const vdm_hier_params* p,
                                           const vdm_analytic* analytic, float* d_grid_out,
                                           vdm_hier_stats* stats, const vdm_hier_debug* debug,
                                           vdm_stream stream) {
    size_t need = 0;
    VDM_TRY(vdm_hierarchical_workspace_size(dec, p, N, &need));
    if (need > kStaticScratchBytes)
        return fail(VDM_ERR_UNSUPPORTED,
                    "this problem needs %zu bytes of scratch; the built-in scratch holds %zu "
                    "(use vdm_decode_hierarchical with a caller workspace)",
                    need, kStaticScratchBytes);
    int dev = 0;
    VDM_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(VDM_ERR_UNSUPPORTED, "device %d out of range", dev);
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_ptr[dev]) {
            void* ptr = nullptr;
            cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
            if (e != cudaSuccess || !ptr)
                return fail(VDM_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
            g_scratch_ptr[dev] = ptr;
        }
        scratch = g_scratch_ptr[dev];
    }
    return vdm_decode_hierarchical(dec, d_k, d_v, B, N, p, analytic, d_grid_out, scratch,
                                   kStaticScratchBytes, stats, debug, stream);
}

}  // extern "C"
