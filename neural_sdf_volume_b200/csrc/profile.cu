// Optional per-launch CUDA-event timing (vdm_profile_begin / vdm_profile_end).
#include <string.h>

#include <vector>

#include "tc_ptx.cuh"
#include "vdm_internal.cuh"

namespace vdm {
namespace {

// the decoder's polynomial 2^x on pairs of elements (the last element of an odd n is paired
// with itself)
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : x0;
    float y0, y1;
    ptx::f32x2_split(ptx::exp2_pair_poly(ptx::f32x2(x0, x1)), y0, y1);
    y[i] = y0;
    if (i + 1 < n) y[i + 1] = y1;
}

struct Rec {
    cudaEvent_t a, b;
    int cls;
};

thread_local bool g_on = false;
thread_local std::vector<Rec> g_recs;
thread_local std::vector<cudaEvent_t> g_pool;
thread_local int64_t g_launch[VDM_PROF_CLASSES];

cudaEvent_t take() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// the decoder's GELU: the pair form that feeds the MLP (bf16) and the scalar form (float32)
__global__ void gelu_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : x0;
    const uint32_t pk = ptx::gelu_as_pack(x0, x1);
    y[i] = __uint_as_float(pk << 16);
    y[n + i] = ptx::gelu_as(x0);
    if (i + 1 < n) {
        y[i + 1] = __uint_as_float(pk & 0xffff0000u);
        y[n + i + 1] = ptx::gelu_as(x1);
    }
}

}  // namespace

void prof_begin(int cls, cudaStream_t s) {
    if (!g_on) return;
    ++g_launch[cls];
    Rec r{take(), take(), cls};
    cudaEventRecord(r.a, s);
    g_recs.push_back(r);
}

void prof_end(int cls, cudaStream_t s) {
    if (!g_on || g_recs.empty()) return;
    (void)cls;
    cudaEventRecord(g_recs.back().b, s);
}

DebugHooks g_debug = {0, 0, 1};   // CTA pairs off by default

}  // namespace vdm

using namespace vdm;

extern "C" {

vdm_status vdm_debug_inject(int32_t mode, int64_t timeout_cycles) {
    if (mode < 0) return fail(VDM_ERR_INVALID_ARG, "inject mode must be >= 0, got %d", mode);
    g_debug.inject = mode;
    g_debug.timeout = timeout_cycles > 0 ? timeout_cycles : 0;
    return VDM_OK;
}

vdm_status vdm_debug_exp2(const float* d_x, float* d_y, int64_t n, vdm_stream stream) {
    if (n < 0) return fail(VDM_ERR_INVALID_ARG, "n must be >= 0, got %lld", (long long)n);
    if (n == 0) return VDM_OK;
    if (!d_x || !d_y) return fail(VDM_ERR_INVALID_ARG, "null array");
    const int64_t pairs = (n + 1) / 2;
    const int64_t blocks = (pairs + 255) / 256;
    if (blocks > 0x7fffffffLL) return fail(VDM_ERR_INVALID_ARG, "n too large: %lld", (long long)n);
    exp2_poly_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(d_x, d_y, n);
    return check_launch("exp2_poly_kernel");
}

vdm_status vdm_debug_gelu(const float* d_x, float* d_y, int64_t n, vdm_stream stream) {
    if (n < 0) return fail(VDM_ERR_INVALID_ARG, "n must be >= 0, got %lld", (long long)n);
    if (n == 0) return VDM_OK;
    if (!d_x || !d_y) return fail(VDM_ERR_INVALID_ARG, "null array");
    const int64_t blocks = ((n + 1) / 2 + 255) / 256;
    if (blocks > 0x7fffffffLL) return fail(VDM_ERR_INVALID_ARG, "n too large: %lld", (long long)n);
    gelu_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(d_x, d_y, n);
    return check_launch("gelu_kernel");
}

vdm_status vdm_set_cta_pairs(int32_t enable) {
    if (enable != 0 && enable != 1) return fail(VDM_ERR_INVALID_ARG, "enable must be 0 or 1, got %d", enable);
    g_debug.single_cta = enable ? 0 : 1;
    return VDM_OK;
}

vdm_status vdm_profile_begin(void) {
    for (auto& r : g_recs) {
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_recs.clear();
    memset(g_launch, 0, sizeof(g_launch));
    g_on = true;
    return VDM_OK;
}

vdm_status vdm_profile_end(vdm_profile* out) {
    if (!out) return fail(VDM_ERR_INVALID_ARG, "out is NULL");
    memset(out, 0, sizeof(*out));
    g_on = false;
    vdm_status st = VDM_OK;
    for (auto& r : g_recs) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
        if (e != cudaSuccess && st == VDM_OK)
            st = fail(VDM_ERR_CUDA, "profile event: %s", cudaGetErrorString(e));
        out->ms[r.cls] += ms;
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_recs.clear();
    for (int c = 0; c < VDM_PROF_CLASSES; ++c) out->launches[c] = g_launch[c];
    return st;
}

}  // extern "C"
