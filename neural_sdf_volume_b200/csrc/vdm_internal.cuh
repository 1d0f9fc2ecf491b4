// Internal declarations of the vecset SDF decoder library (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vdm.h"

namespace vdm {

constexpr int kHeadDim = 64;
constexpr int kPeLanes = 64;
constexpr int kPeDim = 51;
constexpr float kLnEps = 1e-5f;
constexpr int kMaxN = 8192;

// ---------------------------------------------------------------- errors
void set_error(const char* fmt, ...);
vdm_status fail(vdm_status s, const char* fmt, ...);
vdm_status check_launch(const char* what);

#define VDM_CUDA_TRY(expr)                                                              \
    do {                                                                                \
        cudaError_t _e = (expr);                                                        \
        if (_e != cudaSuccess)                                                          \
            return ::vdm::fail(VDM_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(_e)); \
    } while (0)

#define VDM_TRY(expr)                  \
    do {                               \
        vdm_status _s = (expr);        \
        if (_s != VDM_OK) return _s;   \
    } while (0)

// ---------------------------------------------------------------- where queries come from
enum QueryMode : int {
    kQueryGrid = 0,      // query q is voxel q of an R^3 grid
    kQueryXyz = 1,       // query q is xyz[q]
    kQueryChildren = 2,  // query q is child (e & 7) of parent plist[e >> 3], e = q or qorder[q]
};

// Work layout of one decode launch.
enum WorkMode : int {
    kWorkFlat = 0,        // queries [0, M) in fixed-size chunks
    kWorkTileDense = 1,   // per tile: its probes (or all queries of a small tile)
    kWorkTileSparse = 2,  // per tile: its non-probe queries, attention over sel[tile]
};

// Everything a decode kernel needs for one shape (device pointers).
struct DecodeArgs {
    // decoder
    int C, H, F, query_ln;
    const void *Wq, *Wo, *W1, *W2;
    const float *bq, *bo, *b1, *b2, *ln1_g, *ln1_b, *ln2_g, *ln2_b, *w_head, *b_head;
    const float *w_tsdf, *b_tsdf;   // optional tSDF head (NULL: none)
    // keys / values of this shape: [H][N][64]
    const void *K, *V;
    int N;
    // queries
    int qmode;
    int R;                      // grid / children resolution
    const float* xyz;           // kQueryXyz
    const int32_t* plist;       // kQueryChildren: parent linear indices at R/2
    const int32_t* qorder;      // kQueryChildren: optional permutation of children
    const int32_t* qlist;       // kWorkFlat + kQueryChildren: optional slot -> qorder position
    const int32_t* ml_slot;     // with probe_ml in flat work: slot -> probe statistics index
    int64_t M;                  // kWorkFlat: number of queries (upper bound when M_dev is set)
    const int32_t* M_dev;       // kWorkFlat: device-side query count (read by the kernel) or NULL
    // tiles (kWorkTile*)
    int work;
    const int32_t* tile_off;    // [T+1] parent offsets per tile
    int T;
    int n_probe;
    int slots;                  // chunks per tile
    const int32_t* sel;         // [T][ksel]
    int ksel;
    const int32_t* unit_list;   // kWorkTileSparse, single CTAs: the non-empty units (slot * T + tile) or NULL
    const int32_t* n_units_dev; //   and their number (device)
    // outputs
    float* probe_ml;            // kWorkTileDense: per (tile, probe, head) softmax max and sum (log2 units) or NULL
    float* out;                 // out[q] (flat work only) or NULL
    float* grid;                // scatter field at voxel linear index or NULL
    float* dec_grid;            // debug: raw decoder output at voxel index or NULL
    float* tsdf_grid;           // tSDF value at voxel linear index or NULL (needs w_tsdf)
    float* feat_out;            // block output x2[q][C] (fp32) of flat work, or NULL (vecset encoding)
    float* attn_out;            // debug: attention output a[v / attn_stride][C] at voxels v with
    int64_t attn_stride;        //   v % attn_stride == 0 (grid and children modes) or NULL
    // analytic field
    const float* spheres;       // [S][4] or NULL
    int n_spheres;
    float dec_scale;
    float tsdf_trunc;           // tSDF = clip((sphere SDF + dec_scale tanh(t)) / tsdf_trunc, -1, 1)
};

// tSDF value of a query from its raw head output t (analytic term when spheres are given)
__device__ __forceinline__ float tsdf_value(float t, float sphere, const DecodeArgs& a) {
    if (!a.spheres) return t;
    return fminf(1.0f, fmaxf(-1.0f, (sphere + a.dec_scale * tanhf(t)) / a.tsdf_trunc));
}

struct KvArgs {
    int C, H, N;
    const float* z;             // [N][C]
    const void *Wk, *Wv;
    const float *bk, *bv, *g, *b;
    void *K, *V;                // [H][N][64]
};

// SelectArgs: probe points and outputs of adaptive selection (one shape).
struct SelectArgs {
    int C, H, N;
    const void* Wq;
    const float* bq;
    const void* K;              // [H][N][64]
    int T;
    // probe source A: xyz + offsets
    const float* probe_xyz;
    const int32_t* probe_off;   // [T+1]
    // probe source B: hierarchical tiles (first min(n_probe, count) queries of qorder range)
    const int32_t* tile_off;    // [T+1] parent offsets
    const int32_t* tile_list;   // optional: only these tiles (ids into tile_off), else 0..T-1
    const int32_t* plist;
    const int32_t* qorder;
    int R;
    int n_probe;
    int top_k;
    int32_t* sel;               // [T][top_k]
    float* score;               // [T][N] or NULL
};

// ---------------------------------------------------------------- test hooks
struct DebugHooks {
    int inject;              // n >= 1: the n-th tensor-core decode launch from now withholds one signal
    long long timeout;       // bounded-wait limit in cycles (0: default)
    int single_cta;          // 1: tensor-core decoding with one CTA per MMA (no CTA pairs)
};
extern DebugHooks g_debug;

// ---------------------------------------------------------------- profiling
enum ProfClass : int { kProfKv = 0, kProfDecode = 1, kProfSelect = 2, kProfMark = 3, kProfScan = 4,
                       kProfList = 5, kProfFill = 6, kProfProbe = 7 };
void prof_begin(int cls, cudaStream_t s);
void prof_end(int cls, cudaStream_t s);

// ---------------------------------------------------------------- launchers
vdm_status launch_precompute_kv(const KvArgs& a, vdm_dtype dt, cudaStream_t s);
// u[m][C] = W_in pe(points[m]) + b_in (fp32 out; W_in [C][64] in dt)
vdm_status launch_point_features(const float* points, int M, int C, const void* W_in, const float* b_in, float* u,
                                 vdm_dtype dt, cudaStream_t s);
vdm_status launch_decode_simt(const DecodeArgs& a, vdm_dtype dt, int n_ctas_hint, cudaStream_t s);
vdm_status launch_select(const SelectArgs& a, vdm_dtype dt, cudaStream_t s);
// tensor-core decoder (bf16, C in {128, 256, 512}, F % 128 == 0)
bool tc_supported(const DecodeArgs& a, vdm_dtype dt);
vdm_status launch_decode_tc(const DecodeArgs& a, cudaStream_t s);
vdm_status tc_check_error();
constexpr int kTcTile = 128;
// tensor-core probe scoring + Top-K (hierarchical adaptive levels)
struct SelectTcLaunch {
    int C, H, N;
    const void* Wq;
    const float* bq;
    const void* K;              // [H][N][64] bf16
    int T;                      // upper bound of the tiles to score
    const int32_t* n_sel;       // device: tiles to score
    const int32_t* sel_tiles;   // device: their ids
    const int32_t* tile_off;
    const int32_t* plist;
    const int32_t* qorder;
    const float* probe_xyz;     // probes as points [P][3] (or NULL: the first n_probe children in qorder)
    const int32_t* probe_off;   // [T+1] with probe_xyz: tile t's probes, at most n_probe of them
    const float* probe_ml;      // [T][n_probe][H][2] from the dense pass
    int R, n_probe, top_k;
    int32_t* sel;               // [T][top_k]
    float* score_out;           // debug: [score_rows][N] scores of tiles t < score_rows, or NULL
    int score_rows;
};
bool select_tc_supported(int C, int n_probe, int N, vdm_dtype dt);
// probes given as points: statistics row of each probe (t * n_probe + rank), tile list 0..T-1
vdm_status launch_flat_probe_slots(const int32_t* probe_off, int T, int n_probe, int32_t* ml_slot,
                                   int32_t* sel_tiles, int32_t* n_sel, cudaStream_t s);
vdm_status launch_select_tc(const SelectTcLaunch& L, cudaStream_t s);
// picks the kernel for the decoder's dtype and shape; `slots` of tile modes follow its tile size
vdm_status launch_decode(DecodeArgs a, vdm_dtype dt, cudaStream_t s);

// volume kernels
// boundary mark + dilation of a level grid -> blocked refine mask; `bits` is scratch of
// mark_bits_words(R) words
size_t mark_bits_words(int R);
// near-surface bits from |fn| < thr (fn = f for the |f| < 2h rule, the tSDF grid for the tSDF rule)
vdm_status launch_mark_dilate(const float* f, const float* fn, int R, float thr, uint64_t* words, uint64_t* bits,
                              cudaStream_t s);
// voxels with a 26-neighbour of the other sign (no band, no dilation), blocked words
vdm_status launch_sign_change(const float* f, int R, uint64_t* words, uint64_t* bits, cudaStream_t s);
// compaction of the refine mask: word offsets, non-empty word ids (sub-volumes) and
// their parent offsets, parent list, counts[0..1] = refined voxels, sub-volumes;
// `chunk_tmp` is scratch of compact_tmp_ints(n_words) ints
size_t compact_tmp_ints(int n_words);
vdm_status launch_compact(const uint64_t* words, int n_words, int R, int32_t* word_off, int32_t* tile_ids,
                          int32_t* tile_off, int32_t* plist, int32_t* counts, int32_t* chunk_tmp,
                          cudaStream_t s);
// every voxel of the (2R)^3 grid takes its parent's value
vdm_status launch_fill(const float* f_coarse, int R, float* f_fine, cudaStream_t s);
// debug: fine voxel indices of each tile's first min(n_probe, count) queries of qorder
vdm_status launch_probe_export(const int32_t* tile_off, int n_tiles, const int32_t* plist,
                               const int32_t* qorder, int R2, int n_probe, int32_t* out,
                               cudaStream_t s);
// the sparse pass's non-empty (sub-volume, slot) units, `tile_q` queries per slot
vdm_status launch_sparse_units(const int32_t* tile_off, int T, int n_probe, int tile_q, int32_t* list,
                               int32_t* n_units, cudaStream_t s);
vdm_status launch_probe_order(const int32_t* tile_off, int n_tiles, const int32_t* plist, int R2,
                              int n_probe, uint64_t salt, int32_t* qorder, int32_t* counters,
                              int32_t* sel_tiles, int32_t* dense_q, int32_t* dense_ml, cudaStream_t s);


// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load 4 consecutive elements as floats (16-byte aligned for float, 8 for bf16).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// Cell-centred coordinate of index i on an R grid.
__device__ __forceinline__ float grid_coord(int i, int R) {
    return -1.0f + (float)(2 * i + 1) / (float)R;
}

// Fourier embedding lane l (0..63) of point p (lanes >= 51 are zero).
// sin(2^k pi x) is evaluated as sinpi(2^k x): 2^k x is exact in float.
__device__ __forceinline__ float pe_lane(const float p[3], int l) {
    if (l < 3) return p[l];
    if (l < 27) {
        int a = (l - 3) >> 3, k = (l - 3) & 7;
        return sinpif(ldexpf(p[a], k));
    }
    if (l < 51) {
        int a = (l - 27) >> 3, k = (l - 27) & 7;
        return cospif(ldexpf(p[a], k));
    }
    return 0.0f;
}

__device__ __forceinline__ float gelu_erf(float x) {
    return 0.5f * x * (1.0f + erff(x * 0.70710678118654752440f));
}

// Exact SDF of a union of spheres [S][4].
__device__ __forceinline__ float sphere_union(const float p[3], const float* sp, int S) {
    float d = 3.402823466e38f;
    for (int s = 0; s < S; ++s) {
        float dx = p[0] - sp[4 * s], dy = p[1] - sp[4 * s + 1], dz = p[2] - sp[4 * s + 2];
        float r = sqrtf(dx * dx + dy * dy + dz * dz) - sp[4 * s + 3];
        d = fminf(d, r);
    }
    return d;
}

// Child e&7 of parent voxel `par` (linear at R/2) -> fine linear index at R.
__device__ __forceinline__ int64_t child_index(int32_t par, int e, int R) {
    int Rp = R >> 1;
    int i = par / (Rp * Rp), rem = par - i * Rp * Rp;
    int j = rem / Rp, k = rem - j * Rp;
    int fi = 2 * i + ((e >> 2) & 1), fj = 2 * j + ((e >> 1) & 1), fk = 2 * k + (e & 1);
    return ((int64_t)fi * R + fj) * R + fk;
}

__device__ __forceinline__ void voxel_point(int64_t v, int R, float p[3]) {
    int64_t RR = (int64_t)R * R;
    int i = (int)(v / RR);
    int64_t rem = v - (int64_t)i * RR;
    int j = (int)(rem / R), k = (int)(rem - (int64_t)j * R);
    p[0] = grid_coord(i, R);
    p[1] = grid_coord(j, R);
    p[2] = grid_coord(k, R);
}

// SplitMix64 (Steele, Lea & Flood 2014): one step from state x.
__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

}  // namespace vdm
