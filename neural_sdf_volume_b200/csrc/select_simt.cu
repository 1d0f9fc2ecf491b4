// Adaptive KV selection: probe scoring and Top-K per sub-volume.
//
// FlashVDM ("Unleashing Vecset Diffusion Model for Fast Shape Generation",
// aipaper.cc summary, section 4.1 item 2, steps 2-4): a few sampled queries of
// each sub-volume compute their attention to all vecset tokens; the Top-K
// tokens by attention score are kept for the sub-volume.
//
// score[j] = sum over probes p and heads h of softmax_h(q_p K_h^T / 8)_j.
// Each CTA handles one sub-volume: per head, pass 1 finds each probe's softmax
// maximum and normaliser over all tokens (online), pass 2 recomputes the
// logits and adds the normalised weights into score[] (column sums in a fixed
// order: deterministic).  Top-K is a radix select on the float bits (scores
// are >= 0, so bit order is value order) with ties to the smaller token index;
// the kept tokens are written in ascending order.
#include "vdm_internal.cuh"

namespace vdm {
namespace {

constexpr int ST = 256;    // threads
constexpr int PC = 64;     // probes per chunk
constexpr int KB = 64;     // tokens per block
constexpr int LD = 65;     // padded row stride

template <typename T>
__global__ void __launch_bounds__(ST) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) float sm[];
    const int N = a.N, H = a.H;
    float* score = sm;                      // [N]
    float* qh = score + N;                  // [PC][LD]
    float* kb = qh + PC * LD;               // [KB][LD]
    float* pb = kb + KB * LD;               // [PC][LD]
    float* pe = pb + PC * LD;               // [PC][LD]
    float* pts = pe + PC * LD;              // [PC][4]
    uint32_t* keys = reinterpret_cast<uint32_t*>(pts + PC * 4);   // [N] (aliases nothing)
    __shared__ int hist[256];
    __shared__ int wsum[ST / 32];
    __shared__ int red[4];

    const int t = blockIdx.x;
    const int tid = threadIdx.x;
    const T* Kg = static_cast<const T*>(a.K);
    const T* Wq = static_cast<const T*>(a.Wq);

    // ---------------- probes of this sub-volume
    int np;
    int pbase = 0;
    if (a.probe_xyz) {
        pbase = a.probe_off[t];
        np = a.probe_off[t + 1] - pbase;
    } else {
        const int cnt = 8 * (a.tile_off[t + 1] - a.tile_off[t]);
        if (cnt <= a.n_probe) return;   // small sub-volume: decoded densely, no selection
        np = a.n_probe;
        pbase = 8 * a.tile_off[t];
    }
    const int k = a.top_k < N ? a.top_k : N;
    for (int j = tid; j < N; j += ST) score[j] = 0.f;
    __syncthreads();

    const int pr = tid >> 2, tq = tid & 3;   // probe row, token quarter
    for (int c0 = 0; c0 < np; c0 += PC) {
        const int nc = min(PC, np - c0);
        if (tid < PC) {
            float p[3] = {0.f, 0.f, 0.f};
            if (tid < nc) {
                if (a.probe_xyz) {
                    const float* x = a.probe_xyz + (size_t)(pbase + c0 + tid) * 3;
                    p[0] = x[0]; p[1] = x[1]; p[2] = x[2];
                } else {
                    const int e = a.qorder[pbase + c0 + tid];
                    voxel_point(child_index(a.plist[e >> 3], e & 7, a.R), a.R, p);
                }
            }
            pts[tid * 4] = p[0]; pts[tid * 4 + 1] = p[1]; pts[tid * 4 + 2] = p[2];
        }
        __syncthreads();
        for (int i = tid; i < PC * 64; i += ST) {
            const int r = i >> 6, l = i & 63;
            float p[3] = {pts[r * 4], pts[r * 4 + 1], pts[r * 4 + 2]};
            pe[r * LD + l] = pe_lane(p, l);
        }
        __syncthreads();
        for (int h = 0; h < H; ++h) {
            // q_h = Wq[h*64 .. h*64+63] pe + bq  for the chunk's probes
            for (int i = tid; i < PC * 64; i += ST) {
                const int r = i >> 6, d = i & 63;
                const T* w = Wq + (size_t)(h * 64 + d) * kPeLanes;
                float acc = a.bq[h * 64 + d];
                for (int l = 0; l < kPeLanes; l += 4) {
                    const float4 wv = load4(w + l);
                    acc = fmaf(pe[r * LD + l], wv.x, acc);
                    acc = fmaf(pe[r * LD + l + 1], wv.y, acc);
                    acc = fmaf(pe[r * LD + l + 2], wv.z, acc);
                    acc = fmaf(pe[r * LD + l + 3], wv.w, acc);
                }
                qh[r * LD + d] = acc * 0.125f;   // fold the 1/sqrt(64) scale
            }
            // pass 1: running max / normaliser per probe (4 lanes per probe)
            float m_run = -INFINITY, l_run = 0.f;
            for (int pass = 0; pass < 2; ++pass) {
                for (int j0 = 0; j0 < N; j0 += KB) {
                    const int nb = min(KB, N - j0);
                    __syncthreads();
                    for (int i = tid; i < KB * 16; i += ST) {
                        const int jr = i >> 4, d4 = (i & 15) * 4;
                        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (jr < nb) kv = load4(Kg + ((size_t)h * N + j0 + jr) * kHeadDim + d4);
                        float* kd = kb + jr * LD + d4;
                        kd[0] = kv.x; kd[1] = kv.y; kd[2] = kv.z; kd[3] = kv.w;
                    }
                    __syncthreads();
                    float s[16];
                    const float* q = qh + pr * LD;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int j = tq * 16 + i;
                        const float* kr = kb + j * LD;
                        float acc = 0.f;
#pragma unroll 16
                        for (int d = 0; d < 64; ++d) acc = fmaf(q[d], kr[d], acc);
                        s[i] = (j < nb && pr < nc) ? acc : -INFINITY;
                    }
                    if (pass == 0) {
                        float bm = -INFINITY;
#pragma unroll
                        for (int i = 0; i < 16; ++i) bm = fmaxf(bm, s[i]);
                        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
                        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
                        const float m_new = fmaxf(m_run, bm);
                        float ps = 0.f;
                        if (m_new != -INFINITY) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) ps += expf(s[i] - m_new);
                        }
                        ps += __shfl_xor_sync(0xffffffffu, ps, 1);
                        ps += __shfl_xor_sync(0xffffffffu, ps, 2);
                        l_run = (m_run == -INFINITY ? 0.f : l_run * expf(m_run - m_new)) + ps;
                        m_run = m_new;
                    } else {
                        const float inv = pr < nc ? 1.0f / l_run : 0.f;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pb[pr * LD + tq * 16 + i] = pr < nc ? expf(s[i] - m_run) * inv : 0.f;
                        __syncthreads();
                        if (tid < KB && tid < nb) {
                            float cs = 0.f;
                            for (int r = 0; r < PC; ++r) cs += pb[r * LD + tid];
                            score[j0 + tid] += cs;
                        }
                    }
                }
            }
            __syncthreads();
        }
    }
    __syncthreads();
    if (a.score) {
        for (int j = tid; j < N; j += ST) a.score[(size_t)t * N + j] = score[j];
    }
    int32_t* out = a.sel + (size_t)t * a.top_k;
    if (k >= N) {
        for (int j = tid; j < N; j += ST) out[j] = j;
        return;
    }
    // ---------------- radix select of the k-th largest key
    for (int j = tid; j < N; j += ST) keys[j] = __float_as_uint(score[j]);
    uint32_t prefix = 0, pmask = 0;
    int need = k;   // how many of the remaining candidates (matching prefix) to take
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[tid] = 0;
        __syncthreads();
        for (int j = tid; j < N; j += ST) {
            const uint32_t kk = keys[j];
            if ((kk & pmask) == prefix) atomicAdd(&hist[(kk >> shift) & 255], 1);
        }
        __syncthreads();
        if (tid == 0) {
            int acc = 0, b = 255;
            for (; b > 0; --b) {
                if (acc + hist[b] >= need) break;
                acc += hist[b];
            }
            red[0] = b;
            red[1] = need - acc;
        }
        __syncthreads();
        prefix |= (uint32_t)red[0] << shift;
        pmask |= 255u << shift;
        need = red[1];
        __syncthreads();
    }
    const uint32_t thr = prefix;   // k-th largest key; take all > thr and the first `need` == thr
    // flags in index order: each thread owns a contiguous span
    const int per = (N + ST - 1) / ST;
    const int j_lo = tid * per, j_hi = min(N, j_lo + per);
    int eq = 0;
    for (int j = j_lo; j < j_hi; ++j) eq += keys[j] == thr;
    // exclusive scan of eq over threads
    const int lane = tid & 31, warp = tid >> 5;
    int x = eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { const int y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int eq_before = x - eq;
    for (int w = 0; w < warp; ++w) eq_before += wsum[w];
    __syncthreads();
    int take = 0;
    {
        int e = eq_before;
        for (int j = j_lo; j < j_hi; ++j) {
            const uint32_t kk = keys[j];
            const bool tk = kk > thr || (kk == thr && e < need);
            e += kk == thr;
            take += tk;
        }
    }
    x = take;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { const int y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int pos = x - take;
    for (int w = 0; w < warp; ++w) pos += wsum[w];
    {
        int e = eq_before;
        for (int j = j_lo; j < j_hi; ++j) {
            const uint32_t kk = keys[j];
            const bool tk = kk > thr || (kk == thr && e < need);
            e += kk == thr;
            if (tk) out[pos++] = j;
        }
    }
}

}  // namespace

vdm_status launch_select(const SelectArgs& a, vdm_dtype dt, cudaStream_t st) {
    if (a.T <= 0) return VDM_OK;
    const size_t sm = (size_t)(a.N + 3 * PC * LD + KB * LD + PC * 4) * 4 + (size_t)a.N * 4 + 64;
    cudaError_t e = dt == VDM_F32
        ? cudaFuncSetAttribute(select_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)
        : cudaFuncSetAttribute(select_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "select_kernel smem attribute: %s", cudaGetErrorString(e));
    prof_begin(kProfSelect, st);
    if (dt == VDM_F32) {
        select_kernel<float><<<a.T, ST, sm, st>>>(a);
    } else {
        select_kernel<__nv_bfloat16><<<a.T, ST, sm, st>>>(a);
    }
    prof_end(kProfSelect, st);
    return check_launch("select_kernel");
}

}  // namespace vdm
