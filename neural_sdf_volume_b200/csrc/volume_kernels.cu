// Coarse-to-fine volume kernels of hierarchical volume decoding.
//
// FlashVDM ("Unleashing Vecset Diffusion Model for Fast Shape Generation",
// aipaper.cc summary, section 4.1 item 1): after a level is decoded, select the
// voxels whose neighbours change SDF sign, add the near-surface voxels (the
// tSDF threshold rule) and dilate the set once; only the children of the
// selected voxels are decoded at the next resolution, the rest inherit.
//
// Data layout: the refine mask of a level with resolution R (R % 4 == 0) is
// stored blocked, one 64-bit word per 4^3 block of voxels: word
// w = (bi * nb + bj) * nb + bk (nb = R / 4), bit (di * 4 + dj) * 4 + dk.  A word
// is exactly the parent footprint of one aligned 8^3 sub-volume of the next
// level, so per-sub-volume counts are popcounts and the parent list comes out
// grouped by sub-volume ("packing", section 4.1 item 2) with no sort.
#include "vdm_internal.cuh"

namespace vdm {
namespace {

// ------------------------------------------------------------------ mark + dilate
// One CTA covers an 8^3 region (2^3 words).  f is staged with a halo of 2,
// the mark is evaluated on the 10^3 region (halo 1), the dilation on the core.
constexpr int MD_T = 256;
constexpr int MD_E = 12;   // staged edge
constexpr int MM_E = 10;   // mark edge

__global__ void __launch_bounds__(MD_T) mark_dilate_kernel(const float* __restrict__ f, int R,
                                                           float thr, uint64_t* __restrict__ words) {
    __shared__ float fs[MD_E * MD_E * MD_E];
    __shared__ unsigned char ms[MM_E * MM_E * MM_E];
    __shared__ uint32_t half[16];
    const int nb = R >> 2;
    const int ncta = (nb + 1) >> 1;
    int c = blockIdx.x;
    const int ck = c % ncta; c /= ncta;
    const int cj = c % ncta; c /= ncta;
    const int ci = c;
    const int i0 = ci * 8, j0 = cj * 8, k0 = ck * 8;
    for (int t = threadIdx.x; t < MD_E * MD_E * MD_E; t += MD_T) {
        const int a = t / (MD_E * MD_E), b = (t / MD_E) % MD_E, e = t % MD_E;
        const int i = i0 - 2 + a, j = j0 - 2 + b, k = k0 - 2 + e;
        float v = 0.f;
        if (i >= 0 && i < R && j >= 0 && j < R && k >= 0 && k < R)
            v = f[((size_t)i * R + j) * R + k];
        fs[t] = v;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < MM_E * MM_E * MM_E; t += MD_T) {
        const int a = t / (MM_E * MM_E), b = (t / MM_E) % MM_E, e = t % MM_E;
        const int i = i0 - 1 + a, j = j0 - 1 + b, k = k0 - 1 + e;
        unsigned char m = 0;
        if (i >= 0 && i < R && j >= 0 && j < R && k >= 0 && k < R) {
            const float fv = fs[((a + 1) * MD_E + (b + 1)) * MD_E + (e + 1)];
            const bool in = fv < 0.f;
            bool hit = fabsf(fv) < thr;
            for (int da = -1; da <= 1; ++da)
                for (int db = -1; db <= 1; ++db)
                    for (int de = -1; de <= 1; ++de) {
                        const int ni = i + da, nj = j + db, nk = k + de;
                        if (ni < 0 || ni >= R || nj < 0 || nj >= R || nk < 0 || nk >= R) continue;
                        const float fu = fs[((a + 1 + da) * MD_E + (b + 1 + db)) * MD_E + (e + 1 + de)];
                        hit |= ((fu < 0.f) != in);
                    }
            m = hit;
        }
        ms[t] = m;
    }
    __syncthreads();
    // 512 core voxels = 8 words x 64 bits; item -> (word, bit)
    for (int item = threadIdx.x; item < 512; item += MD_T) {
        const int wl = item >> 6, bit = item & 63;
        const int wi = wl >> 2, wj = (wl >> 1) & 1, wk = wl & 1;
        const int di = bit >> 4, dj = (bit >> 2) & 3, dk = bit & 3;
        const int a = wi * 4 + di, b = wj * 4 + dj, e = wk * 4 + dk;   // core coords
        bool act = false;
        for (int da = 0; da < 3; ++da)
            for (int db = 0; db < 3; ++db)
                for (int de = 0; de < 3; ++de)
                    act |= ms[((a + da) * MM_E + (b + db)) * MM_E + (e + de)] != 0;
        const unsigned bal = __ballot_sync(0xffffffffu, act);
        if ((threadIdx.x & 31) == 0) half[item >> 5] = bal;
    }
    __syncthreads();
    if (threadIdx.x < 8) {
        const int wl = threadIdx.x;
        const int bi = ci * 2 + (wl >> 2), bj = cj * 2 + ((wl >> 1) & 1), bk = ck * 2 + (wl & 1);
        if (bi < nb && bj < nb && bk < nb)
            words[((size_t)bi * nb + bj) * nb + bk] =
                (uint64_t)half[2 * wl] | ((uint64_t)half[2 * wl + 1] << 32);
    }
}

// ------------------------------------------------------------------ scan of word popcounts
constexpr int SC_T = 256;
constexpr int SC_PER = 4;
constexpr int SC_BLK = SC_T * SC_PER;   // words per scan block

// Block-wide exclusive scan of (a, b) pairs held one per thread; returns totals.
__device__ __forceinline__ int2 block_scan2(int2 v, int2* tmp, int2& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int2 x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int ya = __shfl_up_sync(0xffffffffu, x.x, o), yb = __shfl_up_sync(0xffffffffu, x.y, o);
        if (lane >= o) { x.x += ya; x.y += yb; }
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int2 w = lane < SC_T / 32 ? tmp[lane] : make_int2(0, 0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int ya = __shfl_up_sync(0xffffffffu, w.x, o), yb = __shfl_up_sync(0xffffffffu, w.y, o);
            if (lane >= o) { w.x += ya; w.y += yb; }
        }
        if (lane < SC_T / 32) tmp[lane] = w;
    }
    __syncthreads();
    int2 base = warp ? tmp[warp - 1] : make_int2(0, 0);
    total = tmp[SC_T / 32 - 1];
    __syncthreads();
    return make_int2(base.x + x.x - v.x, base.y + x.y - v.y);
}

__global__ void __launch_bounds__(SC_T) scan_reduce_kernel(const uint64_t* __restrict__ words, int n,
                                                           int2* __restrict__ bsum) {
    __shared__ int2 tmp[SC_T / 32];
    int2 v = make_int2(0, 0);
    const int base = blockIdx.x * SC_BLK + threadIdx.x * SC_PER;
    for (int q = 0; q < SC_PER; ++q) {
        const int w = base + q;
        if (w < n) {
            const int pc = __popcll(words[w]);
            v.x += pc;
            v.y += pc > 0;
        }
    }
    int2 tot;
    block_scan2(v, tmp, tot);
    if (threadIdx.x == 0) bsum[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(SC_T) scan_blocks_kernel(int2* __restrict__ bsum, int nblk,
                                                           int32_t* __restrict__ counts) {
    __shared__ int2 tmp[SC_T / 32];
    int2 carry = make_int2(0, 0);
    for (int b0 = 0; b0 < nblk; b0 += SC_T) {
        const int b = b0 + threadIdx.x;
        int2 v = b < nblk ? bsum[b] : make_int2(0, 0);
        int2 tot;
        int2 ex = block_scan2(v, tmp, tot);
        if (b < nblk) bsum[b] = make_int2(carry.x + ex.x, carry.y + ex.y);
        carry.x += tot.x;
        carry.y += tot.y;
    }
    if (threadIdx.x == 0) {
        counts[0] = carry.x;   // active parents
        counts[1] = carry.y;   // non-empty words (sub-volumes)
    }
}

__global__ void __launch_bounds__(SC_T) scan_write_kernel(const uint64_t* __restrict__ words, int n,
                                                          const int2* __restrict__ bsum,
                                                          int32_t* __restrict__ word_off,
                                                          int32_t* __restrict__ tile_ids,
                                                          const int32_t* __restrict__ counts) {
    __shared__ int2 tmp[SC_T / 32];
    int pc[SC_PER];
    int2 v = make_int2(0, 0);
    const int base = blockIdx.x * SC_BLK + threadIdx.x * SC_PER;
    for (int q = 0; q < SC_PER; ++q) {
        const int w = base + q;
        pc[q] = w < n ? __popcll(words[w]) : 0;
        v.x += pc[q];
        v.y += pc[q] > 0;
    }
    int2 tot;
    int2 ex = block_scan2(v, tmp, tot);
    const int2 bo = bsum[blockIdx.x];
    int run = bo.x + ex.x, nt = bo.y + ex.y;
    for (int q = 0; q < SC_PER; ++q) {
        const int w = base + q;
        if (w < n) {
            word_off[w] = run;
            if (pc[q] > 0) tile_ids[nt++] = w;
            run += pc[q];
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) word_off[n] = counts[0];
}

// ------------------------------------------------------------------ parent list
__global__ void parent_list_kernel(const uint64_t* __restrict__ words, const int32_t* __restrict__ word_off,
                                   int n, int R, int32_t* __restrict__ plist) {
    const int w = blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= n) return;
    uint64_t m = words[w];
    if (!m) return;
    const int nb = R >> 2;
    const int bi = w / (nb * nb), bj = (w / nb) % nb, bk = w % nb;
    int o = word_off[w];
    while (m) {
        const int bit = __ffsll((long long)m) - 1;
        m &= m - 1;
        const int i = bi * 4 + (bit >> 4), j = bj * 4 + ((bit >> 2) & 3), k = bk * 4 + (bit & 3);
        plist[o++] = (i * R + j) * R + k;
    }
}

__global__ void tile_off_kernel(const int32_t* __restrict__ word_off, const int32_t* __restrict__ tile_ids,
                                int n_tiles, int n_words, int32_t* __restrict__ tile_off) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < n_tiles) tile_off[t] = word_off[tile_ids[t]];
    if (t == n_tiles) tile_off[t] = word_off[n_words];
}

// ------------------------------------------------------------------ inherit fill
// Fine voxels (i, j, 4q..4q+3) at R2 = 2R; parents (i/2, j/2, 2q..2q+1).
__global__ void fill_kernel(const float* __restrict__ fc, const uint64_t* __restrict__ words, int R,
                            float* __restrict__ ff) {
    const int R2 = 2 * R;
    const int Q = R2 >> 2;
    const size_t n = (size_t)R2 * R2 * Q;
    const int nb = R >> 2;
    for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < n; t += (size_t)gridDim.x * blockDim.x) {
        const int q = (int)(t % Q);
        const size_t ij = t / Q;
        const int j = (int)(ij % R2), i = (int)(ij / R2);
        const int pi = i >> 1, pj = j >> 1, pk = 2 * q;
        const size_t pbase = ((size_t)pi * R + pj) * R + pk;
        const float2 pv = *reinterpret_cast<const float2*>(fc + pbase);
        const uint64_t wd = words[((size_t)(pi >> 2) * nb + (pj >> 2)) * nb + (pk >> 2)];
        const int b0 = ((pi & 3) * 4 + (pj & 3)) * 4 + (pk & 3);
        const bool a0 = (wd >> b0) & 1, a1 = (wd >> (b0 + 1)) & 1;
        float* dst = ff + ((size_t)i * R2 + j) * R2 + 4 * q;
        if (!a0 && !a1) {
            *reinterpret_cast<float4*>(dst) = make_float4(pv.x, pv.x, pv.y, pv.y);
        } else {
            if (!a0) { dst[0] = pv.x; dst[1] = pv.x; }
            if (!a1) { dst[2] = pv.y; dst[3] = pv.y; }
        }
    }
}

// ------------------------------------------------------------------ probe order
// Per sub-volume with more than n_probe queries: rank the queries by
// (splitmix64(salt ^ fine_index), fine_index); the n_probe smallest come first
// (in rank order), the rest follow in enumeration order.  Smaller sub-volumes
// keep the identity order (all of their queries are decoded densely).
constexpr int PO_T = 256;
constexpr int PO_MAX = 512;

__global__ void __launch_bounds__(PO_T) probe_order_kernel(const int32_t* __restrict__ tile_off,
                                                           const int32_t* __restrict__ plist, int R2,
                                                           int n_probe, uint64_t salt,
                                                           int32_t* __restrict__ qorder,
                                                           int32_t* __restrict__ counters,
                                                           int32_t* __restrict__ sel_tiles,
                                                           int32_t* __restrict__ dense_q,
                                                           int32_t* __restrict__ dense_ml) {
    __shared__ int dpos;
    __shared__ uint64_t key[PO_MAX];
    __shared__ int wsum[PO_T / 32];
    const int t = blockIdx.x;
    const int base = 8 * tile_off[t];
    const int cnt = 8 * (tile_off[t + 1] - tile_off[t]);
    const int nd = cnt > n_probe ? n_probe : cnt;   // queries decoded over all tokens
    if (threadIdx.x == 0) {   // integer counters: [0] sub-volumes with a selection, [1] full-KV queries
        if (cnt > n_probe) {
            const int pos = atomicAdd(&counters[0], 1);
            if (sel_tiles) sel_tiles[pos] = t;   // list order is irrelevant: each entry is scored alone
        }
        dpos = atomicAdd(&counters[1], nd);
    }
    __syncthreads();
    if (dense_q) {
        // packed list of this sub-volume's full-attention queries (order across
        // sub-volumes is irrelevant: every query is decoded independently)
        for (int i = threadIdx.x; i < nd; i += PO_T) {
            dense_q[dpos + i] = base + i;
            dense_ml[dpos + i] = t * n_probe + i;
        }
    }
    if (cnt <= n_probe) {
        for (int e = threadIdx.x; e < cnt; e += PO_T) qorder[base + e] = base + e;
        return;
    }
    for (int e = threadIdx.x; e < cnt; e += PO_T) {
        const int ge = base + e;
        const int64_t v = child_index(plist[ge >> 3], ge & 7, R2);
        key[e] = splitmix64((uint64_t)v ^ salt);
    }
    __syncthreads();
    // each thread owns two consecutive enumeration slots. Rank = number of smaller keys:
    // the keys are distinct (splitmix64 and the xor with the salt are bijections of the
    // 64-bit words and the voxel indices are distinct), so the rule's tie-break to the
    // smaller voxel never applies. Slots past cnt get the largest key and no position.
    const int e0 = 2 * threadIdx.x;
    const uint64_t k0 = e0 < cnt ? key[e0] : ~0ull, k1 = e0 + 1 < cnt ? key[e0 + 1] : ~0ull;
    int rank[2] = {0, 0};
    for (int f2 = 0; f2 < cnt; ++f2) {
        const uint64_t kf = key[f2];
        rank[0] += kf < k0;
        rank[1] += kf < k1;
    }
    int nonp[2];
    for (int q = 0; q < 2; ++q) nonp[q] = e0 + q < cnt && rank[q] >= n_probe;
    // exclusive scan of the non-probe flags in enumeration order
    const int local = nonp[0] + nonp[1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    int pos = before + x - local;
    for (int q = 0; q < 2; ++q) {
        const int e = 2 * threadIdx.x + q;
        if (e >= cnt) continue;
        if (!nonp[q]) {
            qorder[base + rank[q]] = base + e;
        } else {
            qorder[base + n_probe + pos] = base + e;
            ++pos;
        }
    }
}

}  // namespace

vdm_status launch_mark_dilate(const float* f, int R, uint64_t* words, cudaStream_t s) {
    const int nb = R >> 2, ncta = (nb + 1) >> 1;
    const float thr = (float)(4.0 / (double)R);
    prof_begin(kProfMark, s);
    mark_dilate_kernel<<<ncta * ncta * ncta, MD_T, 0, s>>>(f, R, thr, words);
    prof_end(kProfMark, s);
    return check_launch("mark_dilate_kernel");
}

size_t scan_tmp_ints(int n_words) {
    const int nblk = (n_words + SC_BLK - 1) / SC_BLK;
    return (size_t)2 * nblk + 8;
}

vdm_status launch_word_scan(const uint64_t* words, int n_words, int32_t* word_off, int32_t* tile_ids,
                            int32_t* counts, int32_t* block_tmp, cudaStream_t s) {
    const int nblk = (n_words + SC_BLK - 1) / SC_BLK;
    int2* bsum = reinterpret_cast<int2*>(block_tmp);
    prof_begin(kProfScan, s);
    scan_reduce_kernel<<<nblk, SC_T, 0, s>>>(words, n_words, bsum);
    prof_end(kProfScan, s);
    VDM_TRY(check_launch("scan_reduce_kernel"));
    prof_begin(kProfScan, s);
    scan_blocks_kernel<<<1, SC_T, 0, s>>>(bsum, nblk, counts);
    prof_end(kProfScan, s);
    VDM_TRY(check_launch("scan_blocks_kernel"));
    prof_begin(kProfScan, s);
    scan_write_kernel<<<nblk, SC_T, 0, s>>>(words, n_words, bsum, word_off, tile_ids, counts);
    prof_end(kProfScan, s);
    return check_launch("scan_write_kernel");
}

vdm_status launch_parent_list(const uint64_t* words, const int32_t* word_off, int n_words, int R,
                              int32_t* plist, cudaStream_t s) {
    prof_begin(kProfList, s);
    parent_list_kernel<<<(n_words + 255) / 256, 256, 0, s>>>(words, word_off, n_words, R, plist);
    prof_end(kProfList, s);
    return check_launch("parent_list_kernel");
}

vdm_status launch_tile_offsets(const int32_t* word_off, const int32_t* tile_ids, int n_tiles,
                               int n_words, int32_t* tile_off, cudaStream_t s) {
    prof_begin(kProfList, s);
    tile_off_kernel<<<(n_tiles + 1 + 255) / 256, 256, 0, s>>>(word_off, tile_ids, n_tiles, n_words, tile_off);
    prof_end(kProfList, s);
    return check_launch("tile_off_kernel");
}

vdm_status launch_fill(const float* f_coarse, const uint64_t* words, int R, float* f_fine, cudaStream_t s) {
    const size_t n = (size_t)(2 * R) * (2 * R) * ((2 * R) >> 2);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t want = (n + 255) / 256;
    const int grid = (int)(want < (size_t)sms * 16 ? want : (size_t)sms * 16);
    prof_begin(kProfFill, s);
    fill_kernel<<<grid, 256, 0, s>>>(f_coarse, words, R, f_fine);
    prof_end(kProfFill, s);
    return check_launch("fill_kernel");
}

vdm_status launch_probe_order(const int32_t* tile_off, int n_tiles, const int32_t* plist, int R2,
                              int n_probe, uint64_t salt, int32_t* qorder, int32_t* counters,
                              int32_t* sel_tiles, int32_t* dense_q, int32_t* dense_ml, cudaStream_t s) {
    if (n_tiles <= 0) return VDM_OK;
    prof_begin(kProfProbe, s);
    probe_order_kernel<<<n_tiles, PO_T, 0, s>>>(tile_off, plist, R2, n_probe, salt, qorder, counters, sel_tiles,
                                               dense_q, dense_ml);
    prof_end(kProfProbe, s);
    return check_launch("probe_order_kernel");
}

}  // namespace vdm
