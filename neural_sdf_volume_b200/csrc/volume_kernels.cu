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

// ------------------------------------------------------------------ pack
// Sign and near-surface bits of every voxel, packed into the blocked layout:
// S[w] bit b = f(v) < 0, Nr[w] bit b = |f(v)| < thr.  One CTA per (bi, bj): its
// 16 warps read the 16 rows (4 bi + di, 4 bj + dj) of the block row with 16-byte
// loads (all of a lane's loads in flight at once), each lane turns a float4 into
// the 4-bit nibble (di, dj) of block bk, and the nibbles are gathered into words
// through shared memory.  One read of f, 1/16 of it written.
constexpr int PK_T = 512;          // one warp per row (di, dj)

// MAXV float4 per lane cover rows of up to 128 MAXV voxels; few registers for small
// MAXV keep four CTAs (2048 threads, all loads in flight) on every SM
template <int MAXV>
__global__ void __launch_bounds__(PK_T, MAXV <= 4 ? 4 : 2) pack_kernel(const float* __restrict__ f,
                                                                      const float* __restrict__ fn, int R,
                                                                      float thr, uint64_t* __restrict__ S,
                                                                      uint64_t* __restrict__ Nr) {
    __shared__ __align__(16) uint8_t ns[256][16];   // [bk][row] sign nibbles
    __shared__ __align__(16) uint8_t nn[256][16];   // [bk][row] near nibbles
    const int nb = R >> 2;
    const int bi = blockIdx.x / nb, bj = blockIdx.x - bi * nb;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int di = warp >> 2, dj = warp & 3;
    const size_t roff = ((size_t)(4 * bi + di) * R + (4 * bj + dj)) * R;
    const float4* row = reinterpret_cast<const float4*>(f + roff);
    float4 v[MAXV];
#pragma unroll
    for (int u = 0; u < MAXV; ++u)
        if (lane + 32 * u < nb) v[u] = __ldcs(row + lane + 32 * u);
#pragma unroll
    for (int u = 0; u < MAXV; ++u) {
        const int bk = lane + 32 * u;
        if (bk < nb) {
            const float4 x = v[u];
            ns[bk][warp] = (uint8_t)((x.x < 0.f) | ((x.y < 0.f) << 1) | ((x.z < 0.f) << 2) | ((x.w < 0.f) << 3));
            const float4 y = fn == f ? x : __ldcs(reinterpret_cast<const float4*>(fn + roff) + bk);
            nn[bk][warp] = (uint8_t)((fabsf(y.x) < thr) | ((fabsf(y.y) < thr) << 1) | ((fabsf(y.z) < thr) << 2) |
                                     ((fabsf(y.w) < thr) << 3));
        }
    }
    __syncthreads();
    // thread t < nb: word (bi, bj, t) from its 16 sign nibbles; thread 256 + t: near word
    const int t = threadIdx.x & 255;
    if (t < nb) {
        const uint4 q = *reinterpret_cast<const uint4*>(threadIdx.x < 256 ? ns[t] : nn[t]);
        const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
        uint64_t w = 0;
#pragma unroll
        for (int h = 0; h < 4; ++h) {   // bytes (rows 4h..4h+3, one nibble each) -> 16 bits
            uint32_t x = qq[h];
            x = (x | (x >> 4)) & 0x00FF00FFu;
            x = (x | (x >> 8)) & 0x0000FFFFu;
            w |= (uint64_t)x << (16 * h);
        }
        const size_t wi = ((size_t)bi * nb + bj) * nb + t;
        if (threadIdx.x < 256) S[wi] = w;
        else Nr[wi] = w;
    }
}

// ------------------------------------------------------------------ mark + dilate on words
// mark = near | (D(inside) & D(outside)), act = D(mark), where D is the 3x3x3 dilation
// clipped at the grid border (a voxel's own sign is in its cube, so "some neighbour has
// the other sign" is "the cube holds both signs").  D = D_i o D_j o D_k, and along one
// axis a word's dilation is its shifted copies plus the facing bit planes of its two
// neighbour words.  One CTA computes the act words of an 8^3-word core.  The region it
// stages has a 2-word halo along i and j and a 1-word halo along k (the first k step
// reads the words' k neighbours from global memory): 12 x 12 x 10 words.
constexpr int MW_T = 512;
constexpr int MW_C = 8;                 // core edge (words)
constexpr int MW_EI = MW_C + 4;         // staged extent along i and j
constexpr int MW_EK = MW_C + 2;         // staged extent along k
constexpr int MW_N = MW_EI * MW_EI * MW_EK;
constexpr int MW_SA = MW_EI * MW_EK, MW_SB = MW_EK;   // region strides of i and j
constexpr uint64_t K0 = 0x1111111111111111ull, K3 = 0x8888888888888888ull;   // dk = 0 / 3
constexpr uint64_t J0 = 0x000F000F000F000Full, J3 = 0xF000F000F000F000ull;   // dj = 0 / 3

// one step of the dilation along an axis: x with its shifted copies and the facing bit
// planes of its neighbours xp (minus side) and xn (plus side) along that axis
template <int AXIS>
__device__ __forceinline__ uint64_t dil(uint64_t x, uint64_t xp, uint64_t xn) {
    if (AXIS == 2) return x | ((x >> 1) & ~K3) | ((x << 1) & ~K0) | ((xn & K0) << 3) | ((xp & K3) >> 3);
    if (AXIS == 1) return x | ((x >> 4) & ~J3) | ((x << 4) & ~J0) | ((xn & J0) << 12) | ((xp & J3) >> 12);
    return x | (x >> 16) | (x << 16) | ((xn & 0xFFFFull) << 48) | (xp >> 48);
}

// the same step over staged words (both neighbours inside the region by construction)
template <int AXIS>
__device__ __forceinline__ uint64_t dil_at(const uint64_t* __restrict__ src, int r) {
    constexpr int step = AXIS == 0 ? MW_SA : AXIS == 1 ? MW_SB : 1;
    return dil<AXIS>(src[r], src[r - step], src[r + step]);
}

// visit the region words of the box [A0,A1) x [B0,B1) x [E0,E1) (region coordinates)
template <int A0, int A1, int B0, int B1, int E0, int E1, typename F>
__device__ __forceinline__ void for_box(F f) {
    constexpr int NA = A1 - A0, NB = B1 - B0, NE = E1 - E0;
    for (int t = threadIdx.x; t < NA * NB * NE; t += MW_T) {
        const int e = E0 + t % NE, b = B0 + (t / NE) % NB, a = A0 + t / (NE * NB);
        f(a, b, e, (a * MW_EI + b) * MW_EK + e);
    }
}

// Six passes, each over the box of the region that the passes after it read: (1) load,
// with the k step done from global k neighbours, of the inside and outside words (all
// of the region); (2) j step (b in [1,11)); (3) i step and mark = near | (D(inside) &
// D(outside)) (a, b in [1,11)); then, when dilating, (4) k step (e in [1,9)), (5) j step
// (b in [2,10)) and (6) i step of the mark over the core (a, b in [2,10), e in [1,9)),
// written to the core's words.
template <bool DILATE>
__global__ void __launch_bounds__(MW_T) mark_words_kernel(const uint64_t* __restrict__ S,
                                                          const uint64_t* __restrict__ Nr, int nb,
                                                          uint64_t* __restrict__ act) {
    extern __shared__ uint64_t mw_smem[];
    uint64_t* A = mw_smem;          // D_k(inside), then the mark
    uint64_t* B = A + MW_N;         // D_k(outside), then D_k(mark)
    uint64_t* Nw = B + MW_N;        // near words
    uint64_t* X = Nw + MW_N;        // D_jk(inside), then D_jk(mark)
    uint64_t* Y = X + MW_N;         // D_jk(outside)
    const int ncta = (nb + MW_C - 1) / MW_C;
    int c = blockIdx.x;
    const int ck = c % ncta; c /= ncta;
    const int cj = c % ncta; c /= ncta;
    const int ci = c;
    const int i0 = ci * MW_C - 2, j0 = cj * MW_C - 2, k0 = ck * MW_C - 1;   // region origin (words)
    auto on_grid = [&](int a, int b, int e) -> bool {
        const int bi = i0 + a, bj = j0 + b, bk = k0 + e;
        return bi >= 0 && bi < nb && bj >= 0 && bj < nb && bk >= 0 && bk < nb;
    };
    for_box<0, MW_EI, 0, MW_EI, 0, MW_EK>([&](int a, int b, int e, int r) {
        uint64_t din = 0, dout = 0, n = 0;
        if (on_grid(a, b, e)) {
            const int bk = k0 + e;
            const size_t w = ((size_t)(i0 + a) * nb + (j0 + b)) * nb + bk;
            const uint64_t s = S[w];
            const bool hp = bk > 0, hn = bk + 1 < nb;
            const uint64_t sp = hp ? S[w - 1] : 0ull, sn = hn ? S[w + 1] : 0ull;
            din = dil<2>(s, sp, sn);
            dout = dil<2>(~s, hp ? ~sp : 0ull, hn ? ~sn : 0ull);   // outside words: in-grid only
            n = Nr[w];
        }
        A[r] = din;
        B[r] = dout;
        Nw[r] = n;
    });
    __syncthreads();
    for_box<0, MW_EI, 1, MW_EI - 1, 0, MW_EK>([&](int, int, int, int r) {
        X[r] = dil_at<1>(A, r);
        Y[r] = dil_at<1>(B, r);
    });
    __syncthreads();
    // mark; words off the grid stay empty (their dilated sign words are not)
    for_box<1, MW_EI - 1, 1, MW_EI - 1, 0, MW_EK>([&](int a, int b, int e, int r) {
        A[r] = on_grid(a, b, e) ? (Nw[r] | (dil_at<0>(X, r) & dil_at<0>(Y, r))) : 0ull;
    });
    __syncthreads();
    if (DILATE) {
        for_box<1, MW_EI - 1, 1, MW_EI - 1, 1, MW_EK - 1>([&](int, int, int, int r) { B[r] = dil_at<2>(A, r); });
        __syncthreads();
        for_box<1, MW_EI - 1, 2, MW_EI - 2, 1, MW_EK - 1>([&](int, int, int, int r) { X[r] = dil_at<1>(B, r); });
        __syncthreads();
    }
    for_box<2, MW_EI - 2, 2, MW_EI - 2, 1, MW_EK - 1>([&](int a, int b, int e, int r) {
        const int bi = i0 + a, bj = j0 + b, bk = k0 + e;
        if (bi < nb && bj < nb && bk < nb)
            act[((size_t)bi * nb + bj) * nb + bk] = DILATE ? dil_at<0>(X, r) : A[r];
    });
}

// ------------------------------------------------------------------ compaction
// Chunks of 1024 words in linear word order.  chunk_sum_kernel: per chunk, the number
// of refined voxels and of non-empty words.  compact_kernel: per chunk, the prefix of
// the earlier chunks' sums (each CTA adds them itself: no inter-CTA waiting), then the
// word offsets, the ids and parent offsets of the non-empty words (sub-volumes) and the
// parent list (each word's set bits in ascending bit order, written warp-cooperatively).
constexpr int CP_T = 256;
constexpr int CP_PER = 4;
constexpr int CP_CHUNK = CP_T * CP_PER;

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
        int2 w = lane < CP_T / 32 ? tmp[lane] : make_int2(0, 0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int ya = __shfl_up_sync(0xffffffffu, w.x, o), yb = __shfl_up_sync(0xffffffffu, w.y, o);
            if (lane >= o) { w.x += ya; w.y += yb; }
        }
        if (lane < CP_T / 32) tmp[lane] = w;
    }
    __syncthreads();
    int2 base = warp ? tmp[warp - 1] : make_int2(0, 0);
    total = tmp[CP_T / 32 - 1];
    __syncthreads();
    return make_int2(base.x + x.x - v.x, base.y + x.y - v.y);
}

__device__ __forceinline__ int2 block_sum2(int2 v, int2* tmp) {
    int2 tot;
    block_scan2(v, tmp, tot);
    return tot;
}

__global__ void __launch_bounds__(CP_T) chunk_sum_kernel(const uint64_t* __restrict__ words, int n,
                                                         int2* __restrict__ csum) {
    __shared__ int2 tmp[CP_T / 32];
    int2 v = make_int2(0, 0);
    const int base = blockIdx.x * CP_CHUNK;
    for (int q = 0; q < CP_PER; ++q) {
        const int w = base + q * CP_T + threadIdx.x;   // coalesced: consecutive threads, consecutive words
        if (w < n) {
            const int pc = __popcll(words[w]);
            v.x += pc;
            v.y += pc > 0;
        }
    }
    const int2 tot = block_sum2(v, tmp);
    if (threadIdx.x == 0) csum[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(CP_T) compact_kernel(const uint64_t* __restrict__ words, int n, int R,
                                                       const int2* __restrict__ csum,
                                                       int32_t* __restrict__ word_off,
                                                       int32_t* __restrict__ tile_ids,
                                                       int32_t* __restrict__ tile_off,
                                                       int32_t* __restrict__ plist,
                                                       int32_t* __restrict__ counts) {
    __shared__ int2 tmp[CP_T / 32];
    __shared__ uint64_t sw[CP_CHUNK];
    __shared__ int so[CP_CHUNK];
    const int chunk = blockIdx.x;
    // prefix of the earlier chunks
    int2 pre = make_int2(0, 0);
    for (int c = threadIdx.x; c < chunk; c += CP_T) {
        const int2 x = csum[c];
        pre.x += x.x;
        pre.y += x.y;
    }
    pre = block_sum2(pre, tmp);
    // this thread's CP_PER consecutive words of the chunk
    const int base = chunk * CP_CHUNK;
    const int w0 = base + threadIdx.x * CP_PER;
    uint64_t m[CP_PER];
    int2 v = make_int2(0, 0);
#pragma unroll
    for (int q = 0; q < CP_PER; ++q) {
        m[q] = w0 + q < n ? words[w0 + q] : 0ull;
        const int pc = __popcll(m[q]);
        v.x += pc;
        v.y += pc > 0;
    }
    int2 tot;
    const int2 ex = block_scan2(v, tmp, tot);
    int run = pre.x + ex.x, nt = pre.y + ex.y;
#pragma unroll
    for (int q = 0; q < CP_PER; ++q) {
        const int w = w0 + q;
        const int l = threadIdx.x * CP_PER + q;
        sw[l] = m[q];
        so[l] = run;
        if (w < n) {
            word_off[w] = run;
            if (m[q]) {
                tile_ids[nt] = w;
                tile_off[nt] = run;
                ++nt;
            }
            run += __popcll(m[q]);
        }
    }
    if (base + CP_CHUNK >= n && threadIdx.x == 0) {   // last chunk: totals
        const int total = pre.x + tot.x, T = pre.y + tot.y;
        word_off[n] = total;
        tile_off[T] = total;
        counts[0] = total;   // refined voxels (active parents)
        counts[1] = T;       // non-empty words (sub-volumes)
    }
    __syncthreads();
    if (!plist) return;
    // parent list: each warp takes groups of 32 consecutive words (lane l holds word l of the
    // group, its coordinates and offset); the group's non-empty words are visited by ballot, and
    // for each of them lane L places bits L and L + 32
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbw = R >> 2;
    const uint32_t below = (1u << lane) - 1u;
    for (int g = warp; g < CP_CHUNK / 32; g += CP_T / 32) {
        const int l = g * 32 + lane;
        const int w = base + l;
        const uint64_t x = w < n ? sw[l] : 0ull;
        uint32_t todo = __ballot_sync(0xffffffffu, x != 0ull);
        if (!todo) continue;
        const int bi = w / (nbw * nbw), bj = (w / nbw) % nbw, bk = w % nbw;
        const int corner = ((4 * bi) * R + 4 * bj) * R + 4 * bk;   // linear index of the block's first voxel
        const int o = so[l];
        while (todo) {
            const int src = __ffs(todo) - 1;
            todo &= todo - 1;
            const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)x, src);
            const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(x >> 32), src);
            const int c0 = __shfl_sync(0xffffffffu, corner, src);
            const int o0 = __shfl_sync(0xffffffffu, o, src);
            // bit b = (di * 4 + dj) * 4 + dk -> voxel corner + (di R + dj) R + dk
            if ((lo >> lane) & 1u) {
                const int b = lane;
                plist[o0 + __popc(lo & below)] = c0 + ((b >> 4) * R + ((b >> 2) & 3)) * R + (b & 3);
            }
            if ((hi >> lane) & 1u) {
                const int b = lane + 32;
                plist[o0 + __popc(lo) + __popc(hi & below)] = c0 + ((b >> 4) * R + ((b >> 2) & 3)) * R + (b & 3);
            }
        }
    }
}

// ------------------------------------------------------------------ inherit fill
// Every voxel of the fine grid takes its parent's value (the decode that follows
// overwrites the children of refined parents).  Item t = (coarse row (ci, cj), q): one
// 8-byte load of parents 2q, 2q+1 and one 16-byte store of their 4 children along k in
// each of the 4 fine rows (2ci + di, 2cj + dj); consecutive lanes take consecutive q, so
// every load and store instruction of a warp covers one contiguous span.
template <bool STREAM>
__device__ __forceinline__ void fill_item(const float* __restrict__ fc, int R, float* __restrict__ ff, uint32_t t,
                                          uint32_t Q) {
    const uint32_t cr = t / Q, q = t - cr * Q;
    const uint32_t ci = cr / (uint32_t)R, cj = cr - ci * (uint32_t)R;
    const size_t R2 = 2 * (size_t)R;
    const float2 p = *reinterpret_cast<const float2*>(fc + (size_t)cr * R + 2 * q);
    const float4 v = make_float4(p.x, p.x, p.y, p.y);
    float* row0 = ff + ((2 * ci) * R2 + 2 * cj) * R2 + 4 * q;
#pragma unroll
    for (int d = 0; d < 4; ++d) {
        float4* dst = reinterpret_cast<float4*>(row0 + ((d >> 1) * R2 + (d & 1)) * R2);
        if (STREAM) __stcs(dst, v);
        else *dst = v;
    }
}

template <bool STREAM>
__global__ void __launch_bounds__(256) fill_kernel(const float* __restrict__ fc, int R, float* __restrict__ ff) {
    const uint32_t Q = (uint32_t)R >> 1;                   // parent pairs per coarse row
    const uint32_t n = (uint32_t)R * (uint32_t)R * Q;
    const uint32_t stride = gridDim.x * blockDim.x;
    uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
    for (; t + stride < n; t += 2 * stride) {            // two items in flight per thread
        fill_item<STREAM>(fc, R, ff, t, Q);
        fill_item<STREAM>(fc, R, ff, t + stride, Q);
    }
    if (t < n) fill_item<STREAM>(fc, R, ff, t, Q);
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

// debug export: fine voxel index of each of a tile's first min(n_probe, count) queries in
// the level's query order (its probes, in rank order), -1 after them
__global__ void probe_export_kernel(const int32_t* __restrict__ tile_off, const int32_t* __restrict__ plist,
                                    const int32_t* __restrict__ qorder, int R2, int n_probe,
                                    int32_t* __restrict__ out) {
    const int t = blockIdx.x;
    const int base = 8 * tile_off[t];
    const int cnt = 8 * (tile_off[t + 1] - tile_off[t]);
    const int nd = cnt < n_probe ? cnt : n_probe;
    for (int i = threadIdx.x; i < n_probe; i += blockDim.x) {
        int32_t v = -1;
        if (i < nd) {
            const int e = qorder[base + i];
            v = (int32_t)child_index(plist[e >> 3], e & 7, R2);
        }
        out[(size_t)t * n_probe + i] = v;
    }
}

}  // namespace

vdm_status launch_probe_export(const int32_t* tile_off, int n_tiles, const int32_t* plist,
                               const int32_t* qorder, int R2, int n_probe, int32_t* out, cudaStream_t s) {
    if (n_tiles <= 0) return VDM_OK;
    probe_export_kernel<<<n_tiles, 128, 0, s>>>(tile_off, plist, qorder, R2, n_probe, out);
    return check_launch("probe_export_kernel");
}

vdm_status launch_pack(const float* f, const float* fn, int R, float thr, uint64_t* S, uint64_t* Nr,
                       cudaStream_t s) {
    const int nb = R >> 2;
    if (nb <= 64) pack_kernel<2><<<nb * nb, PK_T, 0, s>>>(f, fn, R, thr, S, Nr);
    else if (nb <= 128) pack_kernel<4><<<nb * nb, PK_T, 0, s>>>(f, fn, R, thr, S, Nr);
    else pack_kernel<8><<<nb * nb, PK_T, 0, s>>>(f, fn, R, thr, S, Nr);
    return check_launch("pack_kernel");
}

size_t mark_bits_words(int R) {
    const size_t nb = (size_t)(R >> 2);
    return 2 * nb * nb * nb;
}

vdm_status launch_mark_dilate(const float* f, const float* fn, int R, float thr, uint64_t* words, uint64_t* bits,
                              cudaStream_t s) {
    if (R % 4 || R < 4 || R > 1024) return fail(VDM_ERR_UNSUPPORTED, "mark: R = %d", R);
    const int nb = R >> 2;
    const size_t nw = (size_t)nb * nb * nb;
    const int smem = 5 * MW_N * (int)sizeof(uint64_t);   // 57.6 KB: set for the current device
    cudaError_t e = cudaFuncSetAttribute(mark_words_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "mark_words smem attribute: %s", cudaGetErrorString(e));
    const int ncta = (nb + MW_C - 1) / MW_C;
    prof_begin(kProfMark, s);
    VDM_TRY(launch_pack(f, fn, R, thr, bits, bits + nw, s));
    mark_words_kernel<true><<<ncta * ncta * ncta, MW_T, smem, s>>>(bits, bits + nw, nb, words);
    prof_end(kProfMark, s);
    return check_launch("mark kernels");
}

vdm_status launch_sign_change(const float* f, int R, uint64_t* words, uint64_t* bits, cudaStream_t s) {
    if (R % 4 || R < 4 || R > 1024) return fail(VDM_ERR_UNSUPPORTED, "sign change: R = %d", R);
    const int nb = R >> 2;
    const size_t nw = (size_t)nb * nb * nb;
    const int smem = 5 * MW_N * (int)sizeof(uint64_t);
    cudaError_t e = cudaFuncSetAttribute(mark_words_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "mark_words smem attribute: %s", cudaGetErrorString(e));
    const int ncta = (nb + MW_C - 1) / MW_C;
    // threshold 0: no near-surface bits, only voxels with a neighbour of the other sign
    VDM_TRY(launch_pack(f, f, R, 0.0f, bits, bits + nw, s));
    mark_words_kernel<false><<<ncta * ncta * ncta, MW_T, smem, s>>>(bits, bits + nw, nb, words);
    return check_launch("sign change kernels");
}

size_t compact_tmp_ints(int n_words) {
    const int nchunk = (n_words + CP_CHUNK - 1) / CP_CHUNK;
    return (size_t)2 * nchunk + 8;
}

vdm_status launch_compact(const uint64_t* words, int n_words, int R, int32_t* word_off, int32_t* tile_ids,
                          int32_t* tile_off, int32_t* plist, int32_t* counts, int32_t* chunk_tmp,
                          cudaStream_t s) {
    const int nchunk = (n_words + CP_CHUNK - 1) / CP_CHUNK;
    int2* csum = reinterpret_cast<int2*>(chunk_tmp);
    prof_begin(kProfScan, s);
    chunk_sum_kernel<<<nchunk, CP_T, 0, s>>>(words, n_words, csum);
    prof_end(kProfScan, s);
    VDM_TRY(check_launch("chunk_sum_kernel"));
    prof_begin(kProfList, s);
    compact_kernel<<<nchunk, CP_T, 0, s>>>(words, n_words, R, csum, word_off, tile_ids, tile_off, plist, counts);
    prof_end(kProfList, s);
    return check_launch("compact_kernel");
}

vdm_status launch_fill(const float* f_coarse, int R, float* f_fine, cudaStream_t s) {
    if (R < 2 || (R & 1)) return fail(VDM_ERR_INVALID_ARG, "fill needs an even resolution (R = %d)", R);
    const size_t n = (size_t)R * R * (R / 2);   // items: 64 bytes of the fine grid each
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t want = (n + 255) / 256;
    const int grid = (int)(want < (size_t)sms * 8 ? want : (size_t)sms * 8);
    if (n + 2 * (size_t)grid * 256 > 0xFFFFFFFFull) return fail(VDM_ERR_UNSUPPORTED, "fill: R = %d too large", R);
    // a fine grid much larger than L2 is written with streaming stores
    const bool stream = n * 64 > ((size_t)64 << 20);
    prof_begin(kProfFill, s);
    if (stream) fill_kernel<true><<<grid, 256, 0, s>>>(f_coarse, R, f_fine);
    else fill_kernel<false><<<grid, 256, 0, s>>>(f_coarse, R, f_fine);
    prof_end(kProfFill, s);
    return check_launch("fill_kernel");
}

// The sparse pass's work units: unit (sub-volume t, slot s) for every slot that holds queries
// (the queries after the first n_probe, 128 per slot), as s * T + t.  The units of a sub-volume
// differ in number, so a static share of all T * slots (unit, slot) pairs per persistent CTA
// gives the CTAs unequal work; a list of the non-empty units shares them evenly.  The order of
// the list does not matter (units are independent).
__global__ void sparse_units_kernel(const int32_t* __restrict__ tile_off, int T, int n_probe, int tile_q,
                                    int32_t* __restrict__ list, int32_t* __restrict__ n_units) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const int cnt = 8 * (tile_off[t + 1] - tile_off[t]);
    const int n = cnt > n_probe ? cnt - n_probe : 0;
    const int units = (n + tile_q - 1) / tile_q;
    if (units == 0) return;
    const int base = atomicAdd(n_units, units);
    for (int sl = 0; sl < units; ++sl) list[base + sl] = sl * T + t;
}

vdm_status launch_sparse_units(const int32_t* tile_off, int T, int n_probe, int tile_q, int32_t* list,
                               int32_t* n_units, cudaStream_t s) {
    VDM_CUDA_TRY(cudaMemsetAsync(n_units, 0, sizeof(int32_t), s));
    if (T <= 0) return VDM_OK;
    sparse_units_kernel<<<(T + 255) / 256, 256, 0, s>>>(tile_off, T, n_probe, tile_q, list, n_units);
    return check_launch("sparse_units_kernel");
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
