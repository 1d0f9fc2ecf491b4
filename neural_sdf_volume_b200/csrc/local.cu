// Local (MSVS-style) vecset decoder query: kNN AVS-Conv on a multi-scale latent
// hierarchy, fused into the SDF.
//
// MSVS-VAE (kwkr.cn article): AVS-Conv (section 1.1) replaces the global
// cross-attention of vecset decoding -- a query point aggregates only its K
// nearest support features, weighted per channel by a small MLP of the
// relative offsets, plus a mean-pooling residual; multi-scale query decoding
// (section 1.3) runs AVS-Conv on every scale of the latent hierarchy and fuses
// the concatenation into the SDF with a light network.
//
//   f_s(x) = (1/K) sum_{j in kNN_s(x)} (w_s(a_j - x) + 1) * F_j,
//   w_s(r) = W2_s GELU(W1_s r + b1_s) + b2_s,
//   sdf(x) = wo . GELU(Wf [f_0, f_1, ...] + bf) + bo.
//
// Neighbours: squared distances in float32, summed x, y then z without fused
// multiply-adds, ties to the smaller anchor index -- the rule decides an index
// set, so it is evaluated exactly as the oracle does.  Search: each scale's
// anchors are binned into a uniform grid over [-1, 1]^3 (anchors outside are
// clamped into the edge cells, which only moves them outward); a query visits
// the cells ring by ring around its own and stops once it holds K neighbours
// whose K-th squared distance lies strictly below the squared distance from
// the query to every cell not yet visited (with a relative margin, so rounding
// can only search one ring more), which makes the result exact.
//
// One thread per query: its kNN in registers, the dynamic-weight hidden layer
// in registers, the scale's channel accumulators in registers, the scale
// outputs in its row of shared memory, then the fusion MLP from shared memory.
// All weights are staged in shared memory once per CTA.
#include <mutex>
#include <string.h>

#include "vdm_internal.cuh"

namespace vdm {
namespace {

constexpr int LQ_T = 64;          // queries per CTA
constexpr int L_MAXS = VDM_LOCAL_MAX_SCALES;
constexpr int L_MAXK = 16, L_MAXH = 32, L_MAXC = 64, L_MAXSUMC = 128, L_MAXF = 64;

struct ScaleGrid {
    int G;                 // cells per axis
    const int32_t* start;  // [G^3 + 1]
    const int32_t* ids;    // [n] anchor ids sorted by cell
};

struct LocalArgs {
    int n_scales, K, hidden, fuse_hidden;
    int C[L_MAXS], coff[L_MAXS], sumC;
    const float* anchors[L_MAXS];
    const float* feats[L_MAXS];
    const float *W1[L_MAXS], *b1[L_MAXS], *W2[L_MAXS], *b2[L_MAXS];
    const float *Wf, *bf, *wo, *bo;
    ScaleGrid grid[L_MAXS];
    const float* xyz;
    int64_t M;
    float* out;
    int32_t* knn_out;      // [M][n_scales][K] or NULL
};

__device__ __forceinline__ int cell_of(float v, int G) {
    int c = (int)floorf((v + 1.0f) * 0.5f * (float)G);
    return c < 0 ? 0 : (c >= G ? G - 1 : c);
}

// ---------------------------------------------------------------- binning
__global__ void bin_count_kernel(const float* __restrict__ a, int n, int G, int32_t* __restrict__ cnt,
                                 int32_t* __restrict__ cell) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int c = (cell_of(a[3 * i], G) * G + cell_of(a[3 * i + 1], G)) * G + cell_of(a[3 * i + 2], G);
    cell[i] = c;
    atomicAdd(&cnt[c], 1);
}

// exclusive scan of the G^3 cell counts (one CTA); start[G^3] = n; cursor = a copy of start
__global__ void __launch_bounds__(1024) bin_scan_kernel(const int32_t* __restrict__ cnt, int nc,
                                                        int32_t* __restrict__ start, int32_t* __restrict__ cursor) {
    __shared__ int ws[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int carry = 0;
    for (int b0 = 0; b0 < nc; b0 += 1024) {
        const int i = b0 + threadIdx.x;
        const int v = i < nc ? cnt[i] : 0;
        int x = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) ws[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = ws[lane];
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            ws[lane] = w;
        }
        __syncthreads();
        const int ex = carry + (warp ? ws[warp - 1] : 0) + x - v;
        if (i < nc) {
            start[i] = ex;
            cursor[i] = ex;
        }
        carry += ws[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) start[nc] = carry;
}

// the order inside a cell does not matter: every anchor of a visited cell is a candidate
// and ties are decided by anchor index
__global__ void bin_place_kernel(const int32_t* __restrict__ cell, int n, int32_t* __restrict__ cursor,
                                 int32_t* __restrict__ ids) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    ids[atomicAdd(&cursor[cell[i]], 1)] = i;
}

// ---------------------------------------------------------------- query
__device__ __forceinline__ float d2_rn(float ax, float ay, float az, float x, float y, float z) {
    const float dx = __fsub_rn(ax, x), dy = __fsub_rn(ay, y), dz = __fsub_rn(az, z);
    return __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
}

// insert (d, id) into the sorted list (d2 ascending, ties by id) of length cnt <= K
__device__ __forceinline__ void knn_insert(float (&bd)[L_MAXK], int (&bi)[L_MAXK], int& cnt, int K, float d,
                                           int id) {
    if (cnt == K && (d > bd[K - 1] || (d == bd[K - 1] && id > bi[K - 1]))) return;
    int p = cnt < K ? cnt : K - 1;
    while (p > 0 && (bd[p - 1] > d || (bd[p - 1] == d && bi[p - 1] > id))) {
        bd[p] = bd[p - 1];
        bi[p] = bi[p - 1];
        --p;
    }
    bd[p] = d;
    bi[p] = id;
    if (cnt < K) ++cnt;
}

__global__ void __launch_bounds__(LQ_T) local_query_kernel(const LocalArgs a) {
    extern __shared__ float lsm[];
    // staged weights: per scale W1, b1, W2, b2; then Wf, bf, wo; then the per-thread feature rows
    float* w1s[L_MAXS];
    float* b1s[L_MAXS];
    float* w2s[L_MAXS];
    float* b2s[L_MAXS];
    float* p = lsm;
    for (int s = 0; s < a.n_scales; ++s) {
        w1s[s] = p; p += a.hidden * 3;
        b1s[s] = p; p += a.hidden;
        w2s[s] = p; p += a.C[s] * a.hidden;
        b2s[s] = p; p += a.C[s];
    }
    float* wfs = p; p += a.fuse_hidden * a.sumC;
    float* bfs = p; p += a.fuse_hidden;
    float* wos = p; p += a.fuse_hidden;
    float* frow = p + threadIdx.x * (a.sumC + 1);   // odd row stride: rows in different banks
    for (int s = 0; s < a.n_scales; ++s) {
        for (int i = threadIdx.x; i < a.hidden * 3; i += LQ_T) w1s[s][i] = a.W1[s][i];
        for (int i = threadIdx.x; i < a.hidden; i += LQ_T) b1s[s][i] = a.b1[s][i];
        for (int i = threadIdx.x; i < a.C[s] * a.hidden; i += LQ_T) w2s[s][i] = a.W2[s][i];
        for (int i = threadIdx.x; i < a.C[s]; i += LQ_T) b2s[s][i] = a.b2[s][i];
    }
    for (int i = threadIdx.x; i < a.fuse_hidden * a.sumC; i += LQ_T) wfs[i] = a.Wf[i];
    for (int i = threadIdx.x; i < a.fuse_hidden; i += LQ_T) {
        bfs[i] = a.bf[i];
        wos[i] = a.wo[i];
    }
    __syncthreads();
    const int64_t q = (int64_t)blockIdx.x * LQ_T + threadIdx.x;
    if (q >= a.M) return;
    const float x = a.xyz[3 * q], y = a.xyz[3 * q + 1], z = a.xyz[3 * q + 2];
    const int K = a.K;
    for (int s = 0; s < a.n_scales; ++s) {
        // ---- exact kNN by rings of cells
        const ScaleGrid g = a.grid[s];
        const float cs = 2.0f / (float)g.G;
        const int cx = cell_of(x, g.G), cy = cell_of(y, g.G), cz = cell_of(z, g.G);
        float bd[L_MAXK];
        int bi[L_MAXK];
        int cnt = 0;
        const float* an = a.anchors[s];
        for (int r = 0; r < g.G; ++r) {
            for (int i = cx - r; i <= cx + r; ++i) {
                if (i < 0 || i >= g.G) continue;
                for (int j = cy - r; j <= cy + r; ++j) {
                    if (j < 0 || j >= g.G) continue;
                    const bool edge_ij = i == cx - r || i == cx + r || j == cy - r || j == cy + r;
                    for (int k = cz - r; k <= cz + r; k += (edge_ij ? 1 : 2 * r > 0 ? 2 * r : 1)) {
                        if (k < 0 || k >= g.G) continue;
                        const int c = (i * g.G + j) * g.G + k;
                        for (int t = g.start[c]; t < g.start[c + 1]; ++t) {
                            const int id = g.ids[t];
                            knn_insert(bd, bi, cnt, K, d2_rn(an[3 * id], an[3 * id + 1], an[3 * id + 2], x, y, z), id);
                        }
                    }
                }
            }
            // unvisited anchors lie beyond a face of the visited box of cells
            float bound = 3.402823466e38f;
            bool all = true;
            const float lox = -1.0f + (float)(cx - r) * cs, hix = -1.0f + (float)(cx + r + 1) * cs;
            const float loy = -1.0f + (float)(cy - r) * cs, hiy = -1.0f + (float)(cy + r + 1) * cs;
            const float loz = -1.0f + (float)(cz - r) * cs, hiz = -1.0f + (float)(cz + r + 1) * cs;
            if (cx - r > 0) { all = false; bound = fminf(bound, x - lox); }
            if (cx + r < g.G - 1) { all = false; bound = fminf(bound, hix - x); }
            if (cy - r > 0) { all = false; bound = fminf(bound, y - loy); }
            if (cy + r < g.G - 1) { all = false; bound = fminf(bound, hiy - y); }
            if (cz - r > 0) { all = false; bound = fminf(bound, z - loz); }
            if (cz + r < g.G - 1) { all = false; bound = fminf(bound, hiz - z); }
            if (all) break;
            // margins: an anchor on a cell face may be binned to either side by rounding
            const float b = bound - 1e-5f;
            if (cnt == K && b > 0.f && bd[K - 1] < b * b * 0.99999f) break;
        }
        if (a.knn_out)
            for (int t = 0; t < K; ++t) a.knn_out[(q * a.n_scales + s) * K + t] = t < cnt ? bi[t] : -1;
        // ---- AVS-Conv of the scale
        const int C = a.C[s];
        float acc[L_MAXC];
#pragma unroll
        for (int c = 0; c < L_MAXC; ++c) acc[c] = 0.f;
        const float* F = a.feats[s];
        for (int t = 0; t < cnt; ++t) {
            const int id = bi[t];
            const float rx = an[3 * id] - x, ry = an[3 * id + 1] - y, rz = an[3 * id + 2] - z;
            float hid[L_MAXH];
#pragma unroll
            for (int h = 0; h < L_MAXH; ++h) {
                if (h < a.hidden) {
                    const float v = w1s[s][3 * h] * rx + w1s[s][3 * h + 1] * ry + w1s[s][3 * h + 2] * rz + b1s[s][h];
                    hid[h] = gelu_erf(v);
                } else {
                    hid[h] = 0.f;
                }
            }
            const float4* Fj = reinterpret_cast<const float4*>(F + (size_t)id * C);
#pragma unroll
            for (int c4 = 0; c4 < L_MAXC / 4; ++c4) {
                if (4 * c4 < C) {
                    const float4 f = Fj[c4];
                    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 4 * c4 + e;
                        float wv = b2s[s][c];
                        const float* w2 = w2s[s] + c * a.hidden;
#pragma unroll
                        for (int h = 0; h < L_MAXH; ++h)
                            if (h < a.hidden) wv = fmaf(w2[h], hid[h], wv);
                        acc[c] = fmaf(wv + 1.0f, fv[e], acc[c]);
                    }
                }
            }
        }
        const float invk = 1.0f / (float)K;
#pragma unroll
        for (int c = 0; c < L_MAXC; ++c)
            if (c < C) frow[a.coff[s] + c] = acc[c] * invk;
    }
    // ---- fusion: wo . GELU(Wf f + bf) + bo
    float sdf = a.bo[0];
    for (int o = 0; o < a.fuse_hidden; ++o) {
        float v = bfs[o];
        const float* wf = wfs + o * a.sumC;
        for (int c = 0; c < a.sumC; ++c) v = fmaf(wf[c], frow[c], v);
        sdf = fmaf(wos[o], gelu_erf(v), sdf);
    }
    a.out[q] = sdf;
}

int grid_cells(int n) {
    int G = 1;
    while ((G + 1) * (G + 1) * (G + 1) * 2 <= n && G < 64) ++G;   // about two anchors per cell
    return G;
}

size_t local_ws_bytes(const vdm_local_decoder* d, size_t* off_cnt, size_t* off_start, size_t* off_cursor,
                      size_t* off_ids, size_t* off_cell) {
    size_t o = 0;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    for (int s = 0; s < d->n_scales; ++s) {
        const size_t G = grid_cells(d->n_anchors[s]);
        const size_t nc = G * G * G;
        off_cnt[s] = o;    o = up(o + nc * 4);
        off_start[s] = o;  o = up(o + (nc + 1) * 4);
        off_cursor[s] = o; o = up(o + nc * 4);
        off_ids[s] = o;    o = up(o + (size_t)d->n_anchors[s] * 4);
        off_cell[s] = o;   o = up(o + (size_t)d->n_anchors[s] * 4);
    }
    return o + 256;
}

vdm_status check_local(const vdm_local_decoder* d) {
    if (!d) return fail(VDM_ERR_INVALID_ARG, "decoder is NULL");
    if (d->n_scales < 1 || d->n_scales > L_MAXS) return fail(VDM_ERR_UNSUPPORTED, "n_scales must be in [1, %d]", L_MAXS);
    if (d->K < 1 || d->K > L_MAXK) return fail(VDM_ERR_UNSUPPORTED, "K must be in [1, %d]", L_MAXK);
    if (d->hidden < 1 || d->hidden > L_MAXH) return fail(VDM_ERR_UNSUPPORTED, "hidden must be in [1, %d]", L_MAXH);
    if (d->fuse_hidden < 1 || d->fuse_hidden > L_MAXF)
        return fail(VDM_ERR_UNSUPPORTED, "fuse_hidden must be in [1, %d]", L_MAXF);
    int sumC = 0;
    for (int s = 0; s < d->n_scales; ++s) {
        if (d->channels[s] < 4 || d->channels[s] > L_MAXC || d->channels[s] % 4)
            return fail(VDM_ERR_UNSUPPORTED, "channels[%d] = %d must be a multiple of 4 in [4, %d]", s, d->channels[s],
                        L_MAXC);
        if (d->n_anchors[s] < d->K || d->n_anchors[s] > (1 << 20))
            return fail(VDM_ERR_UNSUPPORTED, "n_anchors[%d] = %d must be in [K, 2^20]", s, d->n_anchors[s]);
        if (!d->anchors[s] || !d->feats[s] || !d->W1[s] || !d->b1[s] || !d->W2[s] || !d->b2[s])
            return fail(VDM_ERR_INVALID_ARG, "scale %d: null pointer", s);
        if ((uintptr_t)d->feats[s] % 16) return fail(VDM_ERR_INVALID_ARG, "feats[%d] must be 16-byte aligned", s);
        sumC += d->channels[s];
    }
    if (sumC > L_MAXSUMC) return fail(VDM_ERR_UNSUPPORTED, "sum of channels %d > %d", sumC, L_MAXSUMC);
    if (!d->Wf || !d->bf || !d->wo || !d->bo) return fail(VDM_ERR_INVALID_ARG, "null fusion weights");
    return VDM_OK;
}

}  // namespace
}  // namespace vdm

using namespace vdm;

extern "C" {

vdm_status vdm_local_workspace_size(const vdm_local_decoder* d, size_t* bytes) {
    VDM_TRY(check_local(d));
    if (!bytes) return fail(VDM_ERR_INVALID_ARG, "bytes is NULL");
    size_t a[L_MAXS], b[L_MAXS], c[L_MAXS], e[L_MAXS], f[L_MAXS];
    *bytes = local_ws_bytes(d, a, b, c, e, f);
    return VDM_OK;
}

vdm_status vdm_decode_local(const vdm_local_decoder* d, const float* d_xyz, int64_t M, float* d_out,
                            int32_t* d_knn_out, void* d_ws, size_t ws_bytes, vdm_stream stream) {
    size_t need = 0;
    VDM_TRY(vdm_local_workspace_size(d, &need));
    if (M < 0) return fail(VDM_ERR_INVALID_ARG, "M must be >= 0");
    if (M == 0) return VDM_OK;
    if (!d_xyz || !d_out) return fail(VDM_ERR_INVALID_ARG, "null xyz / out");
    if (M > ((int64_t)1 << 31) - 1) return fail(VDM_ERR_UNSUPPORTED, "M too large");
    if (!d_ws || ws_bytes < need) return fail(VDM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    char* ws = reinterpret_cast<char*>(((uintptr_t)d_ws + 255) & ~(uintptr_t)255);
    if ((uintptr_t)ws - (uintptr_t)d_ws + need - 256 > ws_bytes)
        return fail(VDM_ERR_WORKSPACE, "workspace too small after alignment");
    size_t o_cnt[L_MAXS], o_start[L_MAXS], o_cur[L_MAXS], o_ids[L_MAXS], o_cell[L_MAXS];
    local_ws_bytes(d, o_cnt, o_start, o_cur, o_ids, o_cell);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    LocalArgs a;
    memset(&a, 0, sizeof(a));
    a.n_scales = d->n_scales;
    a.K = d->K;
    a.hidden = d->hidden;
    a.fuse_hidden = d->fuse_hidden;
    int sumC = 0;
    for (int s = 0; s < d->n_scales; ++s) {
        a.C[s] = d->channels[s];
        a.coff[s] = sumC;
        sumC += d->channels[s];
        a.anchors[s] = d->anchors[s];
        a.feats[s] = d->feats[s];
        a.W1[s] = d->W1[s]; a.b1[s] = d->b1[s]; a.W2[s] = d->W2[s]; a.b2[s] = d->b2[s];
        // bin the scale's anchors into its grid
        const int n = d->n_anchors[s];
        const int G = grid_cells(n);
        const int nc = G * G * G;
        int32_t* cnt = reinterpret_cast<int32_t*>(ws + o_cnt[s]);
        int32_t* start = reinterpret_cast<int32_t*>(ws + o_start[s]);
        int32_t* cursor = reinterpret_cast<int32_t*>(ws + o_cur[s]);
        int32_t* ids = reinterpret_cast<int32_t*>(ws + o_ids[s]);
        int32_t* cell = reinterpret_cast<int32_t*>(ws + o_cell[s]);
        VDM_CUDA_TRY(cudaMemsetAsync(cnt, 0, (size_t)nc * 4, st));
        bin_count_kernel<<<(n + 255) / 256, 256, 0, st>>>(d->anchors[s], n, G, cnt, cell);
        bin_scan_kernel<<<1, 1024, 0, st>>>(cnt, nc, start, cursor);
        bin_place_kernel<<<(n + 255) / 256, 256, 0, st>>>(cell, n, cursor, ids);
        VDM_TRY(check_launch("local binning kernels"));
        a.grid[s].G = G;
        a.grid[s].start = start;
        a.grid[s].ids = ids;
    }
    a.sumC = sumC;
    a.Wf = d->Wf; a.bf = d->bf; a.wo = d->wo; a.bo = d->bo;
    a.xyz = d_xyz;
    a.M = M;
    a.out = d_out;
    a.knn_out = d_knn_out;
    size_t smem = 0;
    for (int s = 0; s < d->n_scales; ++s) smem += (size_t)(d->hidden * 4 + d->channels[s] * (d->hidden + 1));
    smem += (size_t)d->fuse_hidden * (sumC + 2) + (size_t)LQ_T * (sumC + 1);
    smem *= 4;
    cudaError_t e = cudaFuncSetAttribute(local_query_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "local_query smem attribute: %s", cudaGetErrorString(e));
    local_query_kernel<<<(unsigned)((M + LQ_T - 1) / LQ_T), LQ_T, smem, st>>>(a);
    VDM_TRY(check_launch("local_query_kernel"));
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    return VDM_OK;
}

}  // extern "C"
