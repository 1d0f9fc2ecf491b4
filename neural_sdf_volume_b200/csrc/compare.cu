// Comparison of two SDF volumes on the same grid: the counts behind volume IoU
// (V-IoU) and sign agreement, and the largest absolute difference.
//
// FlashVDM ("Unleashing Vecset Diffusion Model for Fast Shape Generation",
// aipaper.cc summary, section 5 "Evaluation Metrics"; Table 3) judges each
// acceleration of the decoder by the volume IoU of the decoded shape:
// V-IoU = |inside(A) and inside(B)| / |inside(A) or inside(B)|, inside = f < 0.
//
// One pass over both volumes, 16-byte loads, integer counts reduced per warp
// (__reduce_add_sync) and per block, then one 64-bit atomic add per block and
// count: integer sums, so the result is exact and order independent.  The
// maximum of |a - b| is a 64-bit atomic max of the float's bit pattern, which
// orders non-negative floats (a NaN difference sorts above +inf and shows).
#include "vdm_internal.cuh"

namespace vdm {
namespace {

constexpr int CMP_T = 256;

struct Counts {
    uint32_t in_a, in_b, both, same;
    uint32_t dmax;   // float bits of the largest |a - b|
};

__device__ __forceinline__ void account(float a, float b, Counts& c) {
    const bool ia = a < 0.f, ib = b < 0.f;
    c.in_a += ia;
    c.in_b += ib;
    c.both += ia & ib;
    c.same += ia == ib;
    const uint32_t d = __float_as_uint(fabsf(a - b));
    c.dmax = d > c.dmax ? d : c.dmax;
}

template <bool VEC>
__global__ void __launch_bounds__(CMP_T) compare_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                                        int64_t n, unsigned long long* __restrict__ out) {
    Counts c = {0, 0, 0, 0, 0};
    const int64_t stride = (int64_t)gridDim.x * CMP_T;
    const int64_t t0 = (int64_t)blockIdx.x * CMP_T + threadIdx.x;
    if (VEC) {
        const int64_t n4 = n >> 2;
        const float4* a4 = reinterpret_cast<const float4*>(a);
        const float4* b4 = reinterpret_cast<const float4*>(b);
        for (int64_t i = t0; i < n4; i += stride) {
            const float4 x = __ldcs(a4 + i), y = __ldcs(b4 + i);
            account(x.x, y.x, c);
            account(x.y, y.y, c);
            account(x.z, y.z, c);
            account(x.w, y.w, c);
        }
        for (int64_t i = (n4 << 2) + t0; i < n; i += stride) account(a[i], b[i], c);
    } else {
        for (int64_t i = t0; i < n; i += stride) account(a[i], b[i], c);
    }
    __shared__ unsigned long long part[CMP_T / 32][5];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t s0 = __reduce_add_sync(0xffffffffu, c.in_a);
    const uint32_t s1 = __reduce_add_sync(0xffffffffu, c.in_b);
    const uint32_t s2 = __reduce_add_sync(0xffffffffu, c.both);
    const uint32_t s3 = __reduce_add_sync(0xffffffffu, c.same);
    const uint32_t s4 = __reduce_max_sync(0xffffffffu, c.dmax);
    if (lane == 0) {
        part[warp][0] = s0;
        part[warp][1] = s1;
        part[warp][2] = s2;
        part[warp][3] = s3;
        part[warp][4] = s4;
    }
    __syncthreads();
    if (threadIdx.x < 5) {
        unsigned long long v = 0;
        for (int w = 0; w < CMP_T / 32; ++w) {
            const unsigned long long x = part[w][threadIdx.x];
            v = threadIdx.x == 4 ? (x > v ? x : v) : v + x;
        }
        if (threadIdx.x == 4) atomicMax(out + 4, v);
        else atomicAdd(out + threadIdx.x, v);
    }
}

}  // namespace
}  // namespace vdm

using namespace vdm;

extern "C" {

vdm_status vdm_compare_volumes(const float* d_a, const float* d_b, int64_t n, uint64_t* d_out,
                               vdm_stream stream) {
    if (n < 0) return fail(VDM_ERR_INVALID_ARG, "n must be >= 0");
    if (!d_out || (n > 0 && (!d_a || !d_b))) return fail(VDM_ERR_INVALID_ARG, "null a / b / out");
    if ((uintptr_t)d_out % 8) return fail(VDM_ERR_INVALID_ARG, "out must be 8-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    VDM_CUDA_TRY(cudaMemsetAsync(d_out, 0, 5 * sizeof(uint64_t), st));
    if (n == 0) return VDM_OK;
    int dev = 0, sms = 148;
    VDM_CUDA_TRY(cudaGetDevice(&dev));
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // enough resident threads to keep HBM busy: 8 blocks of 256 per SM
    const int64_t want = (n / 4 + CMP_T - 1) / CMP_T;
    const int grid = (int)(want < (int64_t)sms * 8 ? (want > 0 ? want : 1) : (int64_t)sms * 8);
    unsigned long long* out = reinterpret_cast<unsigned long long*>(d_out);
    const bool vec = (uintptr_t)d_a % 16 == 0 && (uintptr_t)d_b % 16 == 0;
    if (vec) compare_kernel<true><<<grid, CMP_T, 0, st>>>(d_a, d_b, n, out);
    else compare_kernel<false><<<grid, CMP_T, 0, st>>>(d_a, d_b, n, out);
    return check_launch("compare_kernel");
}

}  // extern "C"
