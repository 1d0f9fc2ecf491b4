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
// Per chunk of queries: a counting sort of the queries by cell of a 32^3 grid
// (neighbouring threads then walk rings of similar size: the search cost of a
// query grows with its distance to the anchors), then two kernels.
// local_knn_kernel: one thread per query,
// the neighbour list sorted in registers (fixed capacity, static indices); a
// ring of cells is walked through occupancy words staged in shared memory (one
// bit per occupied plane, per occupied row of a plane, per occupied cell of a
// row), so only occupied cells are visited and read from global memory -- a
// query far from every anchor grows its ring many times over empty space.
// local_conv_kernel: one warp per query (lanes over hidden units, channels and
// fusion units; the neighbour's hidden values broadcast by shuffles), all
// weights staged in shared memory once per CTA.
#include <mutex>
#include <string.h>

#include "vdm_internal.cuh"

namespace vdm {
namespace {

constexpr int LQ_T = 256;         // threads per CTA (AVS-Conv and fusion: one warp per query)
constexpr int LK_T = 128;         // queries per CTA (neighbour search)
constexpr int L_CHUNK = 1 << 18;  // queries per chunk (neighbour ids kept in the workspace)
constexpr int L_QG = 32;          // cells per axis of the grid the queries are sorted by
constexpr int L_MAXS = VDM_LOCAL_MAX_SCALES;
constexpr int L_MAXK = 16, L_MAXH = 32, L_MAXC = 64, L_MAXSUMC = 128, L_MAXF = 64;

struct ScaleGrid {
    int G;                 // cells per axis (<= 64)
    const int32_t* start;  // [G^3 + 1]
    const int32_t* ids;    // [n] anchor ids sorted by cell
    const uint64_t* rows;  // [G^2] occupancy of the cells of row (i, j): bit k = cell (i, j, k)
    int row_off;           // offset of the rows in the search kernel's shared memory (words)
};

struct LocalArgs {
    int n_scales, K, hidden, fuse_hidden;
    int C[L_MAXS], coff[L_MAXS], sumC;
    int woff[L_MAXS + 1];  // staged weights: scale s's W1, b1, W2, b2 from woff[s]; the fusion weights at woff[n_scales]
    const float* anchors[L_MAXS];
    const float* feats[L_MAXS];
    const float *W1[L_MAXS], *b1[L_MAXS], *W2[L_MAXS], *b2[L_MAXS];
    const float *Wf, *bf, *wo, *bo;
    ScaleGrid grid[L_MAXS];
    const float* xyz;
    int64_t q0, q1;        // this chunk's queries [q0, q1)
    const int32_t* perm;   // the chunk's queries in cell order: thread t takes query q0 + perm[t]
    float* out;
    int32_t* nbr;          // neighbour ids of query q at nbr[(q - nbr_q0) * n_scales * K]
    int64_t nbr_q0;
    int row_words;         // total occupancy words of all scales
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

// occupancy word of each row of cells
__global__ void row_mask_kernel(const int32_t* __restrict__ cnt, int G, uint64_t* __restrict__ rows) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= G * G) return;
    uint64_t m = 0;
    for (int k = 0; k < G; ++k) m |= (uint64_t)(cnt[r * G + k] > 0) << k;
    rows[r] = m;
}

// ---------------------------------------------------------------- query
__device__ __forceinline__ float d2_rn(float ax, float ay, float az, float x, float y, float z) {
    const float dx = __fsub_rn(ax, x), dy = __fsub_rn(ay, y), dz = __fsub_rn(az, z);
    return __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
}

// (d, id) orders before (e, jd): smaller squared distance, ties to the smaller index
__device__ __forceinline__ bool nb_less(float d, int id, float e, int jd) {
    return d < e || (d == e && id < jd);
}

// insert (d, id) into the sorted list of the KC best (padded with (+inf, INT_MAX));
// every index is static, so the list stays in registers
template <int KC>
__device__ __forceinline__ void knn_insert(float (&bd)[KC], int (&bi)[KC], float d, int id) {
    if (!nb_less(d, id, bd[KC - 1], bi[KC - 1])) return;
#pragma unroll
    for (int p = KC - 1; p > 0; --p) {
        const bool shift = nb_less(d, id, bd[p - 1], bi[p - 1]);
        const bool here = !shift && nb_less(d, id, bd[p], bi[p]);
        bd[p] = shift ? bd[p - 1] : here ? d : bd[p];
        bi[p] = shift ? bi[p - 1] : here ? id : bi[p];
    }
    if (nb_less(d, id, bd[0], bi[0])) {
        bd[0] = d;
        bi[0] = id;
    }
}

// bits lo..hi of a word (0 <= lo <= hi <= 63)
__device__ __forceinline__ uint64_t bit_span(int lo, int hi) {
    return (~0ull >> (63 - hi)) & (~0ull << lo);
}

// Occupancy in shared memory, per scale from row_off: the G^2 row words, then per plane i a
// word with bit j = row (i, j) occupied, then one word with bit i = plane i occupied.  A ring
// visits occupied planes, their occupied rows and those rows' occupied cells only.
template <int KC>
__global__ void __launch_bounds__(LK_T) local_knn_kernel(const LocalArgs a) {
    extern __shared__ uint64_t lrows[];
    for (int s = 0; s < a.n_scales; ++s) {
        const int G = a.grid[s].G;
        uint64_t* r = lrows + a.grid[s].row_off;
        for (int i = threadIdx.x; i < G * G; i += LK_T) r[i] = a.grid[s].rows[i];
    }
    __syncthreads();
    for (int s = 0; s < a.n_scales; ++s) {
        const int G = a.grid[s].G;
        uint64_t* r = lrows + a.grid[s].row_off;
        for (int i = threadIdx.x; i < G; i += LK_T) {
            uint64_t pm = 0;
            for (int j = 0; j < G; ++j) pm |= (uint64_t)(r[i * G + j] != 0) << j;
            r[G * G + i] = pm;
        }
    }
    __syncthreads();
    if (threadIdx.x < a.n_scales) {
        const int G = a.grid[threadIdx.x].G;
        uint64_t* r = lrows + a.grid[threadIdx.x].row_off;
        uint64_t im = 0;
        for (int i = 0; i < G; ++i) im |= (uint64_t)(r[G * G + i] != 0) << i;
        r[G * G + G] = im;
    }
    __syncthreads();
    const int64_t tq = (int64_t)blockIdx.x * LK_T + threadIdx.x;
    if (tq >= a.q1 - a.q0) return;
    const int64_t q = a.q0 + a.perm[tq];
    const float x = a.xyz[3 * q], y = a.xyz[3 * q + 1], z = a.xyz[3 * q + 2];
    const int K = a.K;
    int32_t* nout = a.nbr + (q - a.nbr_q0) * a.n_scales * K;
    for (int s = 0; s < a.n_scales; ++s) {
        const ScaleGrid g = a.grid[s];
        const int G = g.G;
        const uint64_t* rows = lrows + g.row_off;
        const uint64_t* planes = rows + G * G;
        const uint64_t occupied = planes[G];
        const float cs = 2.0f / (float)G;
        const int cx = cell_of(x, G), cy = cell_of(y, G), cz = cell_of(z, G);
        float bd[KC];
        int bi[KC];
#pragma unroll
        for (int p = 0; p < KC; ++p) {
            bd[p] = INFINITY;
            bi[p] = 0x7fffffff;
        }
        int cnt = 0;
        const float* an = a.anchors[s];
        for (int r = 0; r < G; ++r) {
            // ring r: the cells at Chebyshev distance r from the query's cell
            const int i0 = max(cx - r, 0), i1 = min(cx + r, G - 1);
            const int j0 = max(cy - r, 0), j1 = min(cy + r, G - 1);
            const int k0 = max(cz - r, 0), k1 = min(cz + r, G - 1);
            const uint64_t span = (~0ull >> (63 - k1)) & (~0ull << k0);   // k in [k0, k1]
            uint64_t ends = 0;                                              // k = cz - r, cz + r
            if (cz - r >= 0) ends |= 1ull << (cz - r);
            if (cz + r < G) ends |= 1ull << (cz + r);
            const uint64_t jspan = bit_span(j0, j1);
            for (uint64_t iv = occupied & bit_span(i0, i1); iv; iv &= iv - 1) {
                const int i = __ffsll((long long)iv) - 1;
                const bool ei = i == cx - r || i == cx + r;
                for (uint64_t jv = planes[i] & jspan; jv; jv &= jv - 1) {
                    const int j = __ffsll((long long)jv) - 1;
                    uint64_t m = rows[i * G + j] & ((ei || j == cy - r || j == cy + r) ? span : ends);
                    while (m) {
                        const int k = __ffsll((long long)m) - 1;
                        m &= m - 1;
                        const int c = (i * G + j) * G + k;
                        const int t1 = g.start[c + 1];
                        for (int t = g.start[c]; t < t1; ++t) {
                            const int id = g.ids[t];
                            knn_insert<KC>(bd, bi, d2_rn(an[3 * id], an[3 * id + 1], an[3 * id + 2], x, y, z), id);
                            ++cnt;
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
            if (cx + r < G - 1) { all = false; bound = fminf(bound, hix - x); }
            if (cy - r > 0) { all = false; bound = fminf(bound, y - loy); }
            if (cy + r < G - 1) { all = false; bound = fminf(bound, hiy - y); }
            if (cz - r > 0) { all = false; bound = fminf(bound, z - loz); }
            if (cz + r < G - 1) { all = false; bound = fminf(bound, hiz - z); }
            if (all) break;
            if (cnt >= K) {
                float kth = bd[0];
#pragma unroll
                for (int p = 1; p < KC; ++p)
                    if (p == K - 1) kth = bd[p];
                // margins: an anchor on a cell face may be binned to either side by rounding
                const float b = bound - 1e-5f;
                if (b > 0.f && kth < b * b * 0.99999f) break;
            }
        }
#pragma unroll
        for (int p = 0; p < KC; ++p)
            if (p < K) nout[s * K + p] = p < cnt ? bi[p] : -1;
    }
}

// One warp per query.  Lane h computes hidden unit h of a neighbour's dynamic-weight layer
// (hidden <= 32), lanes take channels c = lane and lane + 32 of the per-channel weights and
// features, the scale outputs go to the warp's row in shared memory, then lane o computes
// fusion units o and o + 32.  Weights are staged transposed (W2^T [hidden][C], Wf^T
// [sum C][fuse_hidden]) so that consecutive lanes read consecutive words.
__global__ void __launch_bounds__(LQ_T) local_conv_kernel(const LocalArgs a) {
    extern __shared__ float lsm[];
    const int hd = a.hidden, FH = a.fuse_hidden, SC = a.sumC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int s = 0; s < a.n_scales; ++s) {
        float* w = lsm + a.woff[s];
        const int C = a.C[s];
        for (int i = threadIdx.x; i < hd * 3; i += LQ_T) w[i] = a.W1[s][i];
        for (int i = threadIdx.x; i < hd; i += LQ_T) w[3 * hd + i] = a.b1[s][i];
        for (int i = threadIdx.x; i < C * hd; i += LQ_T) {   // W2 [C][hidden] -> [hidden][C]
            const int c = i / hd, h = i - c * hd;
            w[4 * hd + h * C + c] = a.W2[s][i];
        }
        for (int i = threadIdx.x; i < C; i += LQ_T) w[4 * hd + C * hd + i] = a.b2[s][i];
    }
    float* wft = lsm + a.woff[a.n_scales];   // Wf [FH][SC] -> [SC][FH]
    float* bfs = wft + FH * SC;
    float* wos = bfs + FH;
    float* frow = wos + FH + warp * SC;
    for (int i = threadIdx.x; i < FH * SC; i += LQ_T) {
        const int o = i / SC, c = i - o * SC;
        wft[c * FH + o] = a.Wf[i];
    }
    for (int i = threadIdx.x; i < FH; i += LQ_T) {
        bfs[i] = a.bf[i];
        wos[i] = a.wo[i];
    }
    __syncthreads();
    const int K = a.K;
    const int64_t nq = a.q1 - a.q0;
    const int wpc = LQ_T / 32;
    for (int64_t qi = (int64_t)blockIdx.x * wpc + warp; qi < nq; qi += (int64_t)gridDim.x * wpc) {
        const int64_t q = a.q0 + a.perm[qi];
        const float x = a.xyz[3 * q], y = a.xyz[3 * q + 1], z = a.xyz[3 * q + 2];
        const int32_t* nin = a.nbr + (q - a.nbr_q0) * a.n_scales * K;
        for (int s = 0; s < a.n_scales; ++s) {
            const float* an = a.anchors[s];
            const float* F = a.feats[s];
            const int C = a.C[s];
            const float* w1 = lsm + a.woff[s];
            const float* b1 = w1 + 3 * hd;
            const float* w2t = w1 + 4 * hd;
            const float* b2 = w2t + C * hd;
            const bool c0 = lane < C, c1 = lane + 32 < C;
            const float bias0 = c0 ? b2[lane] : 0.f, bias1 = c1 ? b2[lane + 32] : 0.f;
            const int my_id = lane < K ? nin[s * K + lane] : -1;
            float acc0 = 0.f, acc1 = 0.f;
            for (int t = 0; t < K; ++t) {
                const int id = __shfl_sync(0xffffffffu, my_id, t);
                if (id < 0) continue;
                const float rx = an[3 * id] - x, ry = an[3 * id + 1] - y, rz = an[3 * id + 2] - z;
                const float hv = lane < hd
                    ? gelu_erf(w1[3 * lane] * rx + w1[3 * lane + 1] * ry + w1[3 * lane + 2] * rz + b1[lane])
                    : 0.f;
                const float f0 = c0 ? F[(size_t)id * C + lane] : 0.f;
                const float f1 = c1 ? F[(size_t)id * C + lane + 32] : 0.f;
                float wv0 = bias0, wv1 = bias1;
                for (int h = 0; h < hd; ++h) {
                    const float hh = __shfl_sync(0xffffffffu, hv, h);
                    if (c0) wv0 = fmaf(w2t[h * C + lane], hh, wv0);
                    if (c1) wv1 = fmaf(w2t[h * C + lane + 32], hh, wv1);
                }
                acc0 = fmaf(wv0 + 1.0f, f0, acc0);
                acc1 = fmaf(wv1 + 1.0f, f1, acc1);
            }
            const float invk = 1.0f / (float)K;
            if (c0) frow[a.coff[s] + lane] = acc0 * invk;
            if (c1) frow[a.coff[s] + lane + 32] = acc1 * invk;
        }
        __syncwarp();
        // fusion: wo . GELU(Wf f + bf) + bo
        float part = 0.f;
        for (int o = lane; o < FH; o += 32) {
            float v = bfs[o];
            for (int c = 0; c < SC; ++c) v = fmaf(wft[c * FH + o], frow[c], v);
            part = fmaf(wos[o], gelu_erf(v), part);
        }
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) a.out[q] = a.bo[0] + part;
        __syncwarp();   // frow is rewritten by the warp's next query
    }
}

int grid_cells(int n) {
    int G = 1;
    while ((G + 1) * (G + 1) * (G + 1) * 2 <= n && G < 64) ++G;   // about two anchors per cell
    return G;
}

size_t local_ws_bytes(const vdm_local_decoder* d, size_t* off_cnt, size_t* off_start, size_t* off_cursor,
                      size_t* off_ids, size_t* off_cell, size_t* off_rows, size_t* off_nbr, size_t* off_q) {
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
        off_rows[s] = o;   o = up(o + G * G * 8);
    }
    *off_nbr = o;          // neighbour ids of one chunk of queries
    o = up(o + (size_t)L_CHUNK * d->n_scales * d->K * 4);
    off_q[0] = o;          // query cells of a chunk
    o = up(o + (size_t)L_CHUNK * 4);
    off_q[1] = o;          // the chunk's order
    o = up(o + (size_t)L_CHUNK * 4);
    const size_t nqc = (size_t)L_QG * L_QG * L_QG;
    off_q[2] = o; o = up(o + nqc * 4);          // counts
    off_q[3] = o; o = up(o + (nqc + 1) * 4);    // starts
    off_q[4] = o; o = up(o + nqc * 4);          // cursors
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
    size_t a[L_MAXS], b[L_MAXS], c[L_MAXS], e[L_MAXS], f[L_MAXS], g[L_MAXS], h, qo[5];
    *bytes = local_ws_bytes(d, a, b, c, e, f, g, &h, qo);
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
    size_t o_cnt[L_MAXS], o_start[L_MAXS], o_cur[L_MAXS], o_ids[L_MAXS], o_cell[L_MAXS], o_rows[L_MAXS], o_nbr,
        o_q[5];
    local_ws_bytes(d, o_cnt, o_start, o_cur, o_ids, o_cell, o_rows, &o_nbr, o_q);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    LocalArgs a;
    memset(&a, 0, sizeof(a));
    a.n_scales = d->n_scales;
    a.K = d->K;
    a.hidden = d->hidden;
    a.fuse_hidden = d->fuse_hidden;
    int sumC = 0, row_words = 0;
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
        uint64_t* rows = reinterpret_cast<uint64_t*>(ws + o_rows[s]);
        VDM_CUDA_TRY(cudaMemsetAsync(cnt, 0, (size_t)nc * 4, st));
        bin_count_kernel<<<(n + 255) / 256, 256, 0, st>>>(d->anchors[s], n, G, cnt, cell);
        bin_scan_kernel<<<1, 1024, 0, st>>>(cnt, nc, start, cursor);
        bin_place_kernel<<<(n + 255) / 256, 256, 0, st>>>(cell, n, cursor, ids);
        row_mask_kernel<<<(G * G + 255) / 256, 256, 0, st>>>(cnt, G, rows);
        VDM_TRY(check_launch("local binning kernels"));
        a.grid[s].G = G;
        a.grid[s].start = start;
        a.grid[s].ids = ids;
        a.grid[s].rows = rows;
        a.grid[s].row_off = row_words;
        row_words += G * G + G + 1;
    }
    a.sumC = sumC;
    a.row_words = row_words;
    a.Wf = d->Wf; a.bf = d->bf; a.wo = d->wo; a.bo = d->bo;
    a.xyz = d_xyz;
    a.out = d_out;
    const size_t ksmem = (size_t)row_words * 8;
    auto knn = d->K <= 8 ? local_knn_kernel<8> : local_knn_kernel<16>;
    cudaError_t e = cudaFuncSetAttribute(knn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ksmem);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "local_knn smem attribute: %s", cudaGetErrorString(e));
    size_t smem = 0;
    for (int s = 0; s < d->n_scales; ++s) {
        a.woff[s] = (int)smem;
        smem += (size_t)(d->hidden * 4 + d->channels[s] * (d->hidden + 1));
    }
    a.woff[d->n_scales] = (int)smem;
    smem += (size_t)d->fuse_hidden * (sumC + 2) + (size_t)(LQ_T / 32) * sumC;
    smem *= 4;
    e = cudaFuncSetAttribute(local_conv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "local_conv smem attribute: %s", cudaGetErrorString(e));
    // with d_knn_out the neighbour ids go straight to it; else through the workspace, chunk by chunk
    for (int64_t q0 = 0; q0 < M; q0 += L_CHUNK) {
        a.q0 = q0;
        a.q1 = q0 + L_CHUNK < M ? q0 + L_CHUNK : M;
        a.nbr = d_knn_out ? d_knn_out : reinterpret_cast<int32_t*>(ws + o_nbr);
        a.nbr_q0 = d_knn_out ? 0 : q0;
        const unsigned nq = (unsigned)(a.q1 - a.q0);
        // sort the chunk's queries by cell: neighbouring threads then walk similar rings
        int32_t* qcell = reinterpret_cast<int32_t*>(ws + o_q[0]);
        int32_t* perm = reinterpret_cast<int32_t*>(ws + o_q[1]);
        int32_t* qcnt = reinterpret_cast<int32_t*>(ws + o_q[2]);
        int32_t* qstart = reinterpret_cast<int32_t*>(ws + o_q[3]);
        int32_t* qcur = reinterpret_cast<int32_t*>(ws + o_q[4]);
        const int nqc = L_QG * L_QG * L_QG;
        VDM_CUDA_TRY(cudaMemsetAsync(qcnt, 0, (size_t)nqc * 4, st));
        bin_count_kernel<<<(nq + 255) / 256, 256, 0, st>>>(d_xyz + 3 * q0, (int)nq, L_QG, qcnt, qcell);
        bin_scan_kernel<<<1, 1024, 0, st>>>(qcnt, nqc, qstart, qcur);
        bin_place_kernel<<<(nq + 255) / 256, 256, 0, st>>>(qcell, (int)nq, qcur, perm);
        a.perm = perm;
        knn<<<(nq + LK_T - 1) / LK_T, LK_T, ksmem, st>>>(a);
        const unsigned conv_ctas = (nq + LQ_T / 32 - 1) / (LQ_T / 32);
        local_conv_kernel<<<conv_ctas < 148u * 8u ? conv_ctas : 148u * 8u, LQ_T, smem, st>>>(a);
        VDM_TRY(check_launch("local query kernels"));
    }
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    return VDM_OK;
}

}  // extern "C"
