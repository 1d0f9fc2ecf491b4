// Surface extraction from a decoded SDF volume: marching cubes restricted to
// the cubes that meet the surface.
//
// The last stage of the shape pipeline turns the decoded volume into a mesh
// (techwalker article, section 1: image encoding -> diffusion sampling -> VAE
// decoding -> surface extraction).  Marching cubes on the grid of decoded
// samples: a cube of 2^3 neighbouring samples whose corners have both signs
// holds polygons whose vertices sit on its edges where the field crosses zero.
//
// Sparse: a cube with both signs has corners with a 26-neighbour of the other
// sign, so the cubes to visit are those touching a "sign-change" voxel.  The
// sign-change voxels are found with the same bit-parallel word kernels as the
// boundary marking of hierarchical decoding (no band, no dilation), and only
// 8^3-cube blocks near them are visited: the result equals marching cubes over
// every cube of the grid, for any input.
//
// Conventions (inside f < 0; corner c = 4 ci + 2 cj + ck; edge e = 4 a + 2 u + v
// along axis a between the corners whose other two coordinates are (u, v)):
//   * a face with two sign changes gets one segment between its crossed edges;
//     with four, two segments that each cut off one inside corner;
//   * a segment A -> B is oriented so that an inside corner P of its side has
//     ((B - A) x (P - A)) . n < 0 (n the face's outward normal, edge midpoints
//     for A and B); segments chain into loops, each listed from its smallest
//     edge, loops by smallest edge; a loop is fanned from its first vertex (in
//     loop order) none of whose fan diagonals joins two edges of one face;
//     normals point to f > 0;
//   * the crossed edge from sample p0 to p0 + 1 along axis a holds the vertex
//     p0 + t h e_a, t = f0 / (f0 - f1), and belongs to sample p0;
//   * samples and cubes (by minimum corner) are ordered by 8^3 block (linear
//     block order), then linear order inside the block; a sample's vertices
//     in axis order; triangles cube by cube in loop and fan order.
// The 256-entry case table is generated on the host from these rules.
#include <math.h>
#include <mutex>
#include <string.h>

#include "vdm_internal.cuh"

namespace vdm {
namespace {

constexpr int MC_MAXT = 5;     // triangles per cube (the rules above never give more)
constexpr int MC_T = 512;      // one thread per sample / cube of an 8^3 block

struct McTable {
    uint8_t ntri[256];
    uint8_t tri[256][MC_MAXT][3];   // edge ids
};

__constant__ McTable c_mc;

// ---------------------------------------------------------------- case table (host)
struct V3 {
    double x[3];
};
V3 corner_pos(int c) { return V3{{(double)((c >> 2) & 1), (double)((c >> 1) & 1), (double)(c & 1)}}; }
void edge_corners(int e, int& c0, int& c1) {
    const int a = e / 4, u = (e >> 1) & 1, v = e & 1;
    int lo[3] = {0, 0, 0}, o = 0;
    for (int x = 0; x < 3; ++x)
        if (x != a) lo[x] = (o++ == 0) ? u : v;
    c0 = 4 * lo[0] + 2 * lo[1] + lo[2];
    c1 = c0 | (1 << (2 - a));
}
V3 edge_mid(int e) {
    int c0, c1;
    edge_corners(e, c0, c1);
    const V3 p = corner_pos(c0), q = corner_pos(c1);
    return V3{{(p.x[0] + q.x[0]) / 2, (p.x[1] + q.x[1]) / 2, (p.x[2] + q.x[2]) / 2}};
}
int edge_between(int c0, int c1) {
    const V3 p = corner_pos(c0), q = corner_pos(c1);
    int a = 0;
    while (p.x[a] == q.x[a]) ++a;
    int uv[2], o = 0;
    for (int x = 0; x < 3; ++x)
        if (x != a) uv[o++] = (int)p.x[x];
    return 4 * a + 2 * uv[0] + uv[1];
}
// faces of an edge as bits (axis a, side s) -> bit 2 a + s
int edge_faces(int e) {
    int c0, c1;
    edge_corners(e, c0, c1);
    const V3 p = corner_pos(c0), q = corner_pos(c1);
    int m = 0;
    for (int a = 0; a < 3; ++a)
        if (p.x[a] == q.x[a]) m |= 1 << (2 * a + (int)p.x[a]);
    return m;
}

bool build_table(McTable& t) {
    memset(&t, 0, sizeof(t));
    for (int cfg = 0; cfg < 256; ++cfg) {
        auto inside = [&](int c) { return ((cfg >> c) & 1) != 0; };
        int nxt[12];
        for (int e = 0; e < 12; ++e) nxt[e] = -1;
        for (int a = 0; a < 3; ++a) {
            int oth[2], o = 0;
            for (int x = 0; x < 3; ++x)
                if (x != a) oth[o++] = x;
            for (int s = 0; s < 2; ++s) {
                // corners of the face in cyclic order
                int cyc[4];
                const int uv[4][2] = {{0, 0}, {1, 0}, {1, 1}, {0, 1}};
                for (int q = 0; q < 4; ++q) {
                    int p[3];
                    p[a] = s;
                    p[oth[0]] = uv[q][0];
                    p[oth[1]] = uv[q][1];
                    cyc[q] = 4 * p[0] + 2 * p[1] + p[2];
                }
                int crossed[4], nc = 0;
                for (int q = 0; q < 4; ++q)
                    if (inside(cyc[q]) != inside(cyc[(q + 1) % 4])) crossed[nc++] = edge_between(cyc[q], cyc[(q + 1) % 4]);
                int seg[2][3], ns = 0;
                if (nc == 2) {
                    int pin = -1;
                    for (int q = 0; q < 4 && pin < 0; ++q)
                        if (inside(cyc[q])) pin = cyc[q];
                    seg[0][0] = crossed[0];
                    seg[0][1] = crossed[1];
                    seg[0][2] = pin;
                    ns = 1;
                } else if (nc == 4) {
                    for (int q = 0; q < 4; ++q)
                        if (inside(cyc[q])) {
                            seg[ns][0] = edge_between(cyc[(q + 3) % 4], cyc[q]);
                            seg[ns][1] = edge_between(cyc[q], cyc[(q + 1) % 4]);
                            seg[ns][2] = cyc[q];
                            ++ns;
                        }
                }
                double n[3] = {0, 0, 0};
                n[a] = s ? 1.0 : -1.0;
                for (int g = 0; g < ns; ++g) {
                    int ea = seg[g][0], eb = seg[g][1];
                    const V3 A = edge_mid(ea), B = edge_mid(eb), P = corner_pos(seg[g][2]);
                    const double u[3] = {B.x[0] - A.x[0], B.x[1] - A.x[1], B.x[2] - A.x[2]};
                    const double w[3] = {P.x[0] - A.x[0], P.x[1] - A.x[1], P.x[2] - A.x[2]};
                    const double cr[3] = {u[1] * w[2] - u[2] * w[1], u[2] * w[0] - u[0] * w[2],
                                          u[0] * w[1] - u[1] * w[0]};
                    if (cr[0] * n[0] + cr[1] * n[1] + cr[2] * n[2] > 0) {
                        const int x = ea;
                        ea = eb;
                        eb = x;
                    }
                    if (nxt[ea] >= 0) return false;   // two segments leave one edge
                    nxt[ea] = eb;
                }
            }
        }
        bool seen[12] = {};
        int nt = 0;
        for (int st = 0; st < 12; ++st) {
            if (nxt[st] < 0 || seen[st]) continue;
            int loop[12], m = 0;
            int e = st;
            do {
                if (m == 12) return false;
                loop[m++] = e;
                seen[e] = true;
                e = nxt[e];
            } while (e != st && e >= 0);
            if (e != st || m < 3) return false;
            int apex = -1;
            for (int sh = 0; sh < m && apex < 0; ++sh) {
                bool ok = true;
                for (int q = 2; q <= m - 2; ++q)
                    if (edge_faces(loop[sh]) & edge_faces(loop[(sh + q) % m])) ok = false;
                if (ok) apex = sh;
            }
            if (apex < 0) return false;
            for (int q = 1; q <= m - 2; ++q) {
                if (nt == MC_MAXT) return false;
                t.tri[cfg][nt][0] = (uint8_t)loop[apex];
                t.tri[cfg][nt][1] = (uint8_t)loop[(apex + q) % m];
                t.tri[cfg][nt][2] = (uint8_t)loop[(apex + q + 1) % m];
                ++nt;
            }
        }
        t.ntri[cfg] = (uint8_t)nt;
    }
    return true;
}

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ bool word_set(const uint64_t* __restrict__ words, int nw1, int wi, int wj, int wk) {
    return wi >= 0 && wi < nw1 && wj >= 0 && wj < nw1 && wk >= 0 && wk < nw1 &&
           words[((size_t)wi * nw1 + wj) * nw1 + wk] != 0ull;
}

// a block of 8^3 cubes must be visited when a sign-change word lies within
// [2b - 2, 2b + 2] per axis: its cubes' corners span words [2b, 2b + 2], and its
// samples own edges of cubes of the blocks b - 1 too
__global__ void mc_flag_kernel(const uint64_t* __restrict__ chg, int R, uint64_t* __restrict__ flag) {
    const int nb8 = R >> 3, nw1 = R >> 2;
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= nb8 * nb8 * nb8) return;
    const int bi = b / (nb8 * nb8), bj = (b / nb8) % nb8, bk = b % nb8;
    bool any = false;
    for (int di = -2; di <= 2 && !any; ++di)
        for (int dj = -2; dj <= 2 && !any; ++dj)
            for (int dk = -2; dk <= 2 && !any; ++dk)
                any = word_set(chg, nw1, 2 * bi + di, 2 * bj + dj, 2 * bk + dk);
    flag[b] = any ? 1ull : 0ull;
}

struct Block {
    int R, i0, j0, k0;
};

// sample (i, j, k): number of its own crossed edges (axes a with a + 1 sample)
__device__ __forceinline__ int own_edges(const float* __restrict__ f, int R, int i, int j, int k, int below_axis,
                                         float f0) {
    const bool in0 = f0 < 0.f;
    const size_t s = ((size_t)i * R + j) * R + k;
    int n = 0;
    if (below_axis > 0 && i + 1 < R) n += (f[s + (size_t)R * R] < 0.f) != in0;
    if (below_axis > 1 && j + 1 < R) n += (f[s + R] < 0.f) != in0;
    if (below_axis > 2 && k + 1 < R) n += (f[s + 1] < 0.f) != in0;
    return n;
}

__device__ __forceinline__ int cube_config(const float* __restrict__ f, int R, int i, int j, int k) {
    int cfg = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const int ci = (c >> 2) & 1, cj = (c >> 1) & 1, ck = c & 1;
        cfg |= (f[((size_t)(i + ci) * R + (j + cj)) * R + (k + ck)] < 0.f) << c;
    }
    return cfg;
}

// block-wide exclusive scan of (a, b) over MC_T threads
__device__ __forceinline__ int2 mc_scan2(int2 v, int2* tmp, int2& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int2 x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, x.x, o), yb = __shfl_up_sync(0xffffffffu, x.y, o);
        if (lane >= o) {
            x.x += ya;
            x.y += yb;
        }
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int2 w = lane < MC_T / 32 ? tmp[lane] : make_int2(0, 0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ya = __shfl_up_sync(0xffffffffu, w.x, o), yb = __shfl_up_sync(0xffffffffu, w.y, o);
            if (lane >= o) {
                w.x += ya;
                w.y += yb;
            }
        }
        if (lane < MC_T / 32) tmp[lane] = w;
    }
    __syncthreads();
    const int2 base = warp ? tmp[warp - 1] : make_int2(0, 0);
    total = tmp[MC_T / 32 - 1];
    __syncthreads();
    return make_int2(base.x + x.x - v.x, base.y + x.y - v.y);
}

// band: the block's cubes have a corner in a sign-change word ([2b, 2b + 2] per axis)
__device__ __forceinline__ bool block_band(const uint64_t* __restrict__ chg, int R, int bi, int bj, int bk) {
    bool any = false;
    if (threadIdx.x < 27) {
        const int d = threadIdx.x;
        any = word_set(chg, R >> 2, 2 * bi + d / 9, 2 * bj + (d / 3) % 3, 2 * bk + d % 3);
    }
    return __syncthreads_or(any) != 0;
}

__global__ void __launch_bounds__(MC_T) mc_count_kernel(const float* __restrict__ f, int R,
                                                        const uint64_t* __restrict__ chg,
                                                        const int32_t* __restrict__ n_slots,
                                                        const int32_t* __restrict__ slot_block,
                                                        uint16_t* __restrict__ vloc, int2* __restrict__ btot) {
    __shared__ int2 tmp[MC_T / 32];
    const int n = *n_slots;
    const int nb8 = R >> 3;
    for (int slot = blockIdx.x; slot < n; slot += gridDim.x) {   // uniform across the CTA
        const int b = slot_block[slot];
        const int bi = b / (nb8 * nb8), bj = (b / nb8) % nb8, bk = b % nb8;
        const bool band = block_band(chg, R, bi, bj, bk);
        const int l = threadIdx.x;
        const int i = 8 * bi + (l >> 6), j = 8 * bj + ((l >> 3) & 7), k = 8 * bk + (l & 7);
        const float f0 = f[((size_t)i * R + j) * R + k];
        int2 v;
        v.x = own_edges(f, R, i, j, k, 3, f0);
        v.y = (band && i + 1 < R && j + 1 < R && k + 1 < R) ? c_mc.ntri[cube_config(f, R, i, j, k)] : 0;
        int2 tot;
        const int2 ex = mc_scan2(v, tmp, tot);
        vloc[(size_t)slot * MC_T + l] = (uint16_t)ex.x;
        if (l == 0) btot[slot] = tot;
    }
}

// exclusive scan of the per-block totals (one CTA); out[0..1] = vertices, triangles
__global__ void __launch_bounds__(1024) mc_scan_kernel(const int2* __restrict__ btot, const int32_t* __restrict__ n_slots,
                                                       int2* __restrict__ bpre, long long* __restrict__ out) {
    __shared__ long long wa[32], wb[32];
    const int n = *n_slots;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long ca = 0, cb = 0;
    for (int s0 = 0; s0 < n; s0 += 1024) {
        const int s = s0 + threadIdx.x;
        const int2 v = s < n ? btot[s] : make_int2(0, 0);
        long long xa = v.x, xb = v.y;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long ya = __shfl_up_sync(0xffffffffu, xa, o), yb = __shfl_up_sync(0xffffffffu, xb, o);
            if (lane >= o) {
                xa += ya;
                xb += yb;
            }
        }
        if (lane == 31) {
            wa[warp] = xa;
            wb[warp] = xb;
        }
        __syncthreads();
        if (warp == 0) {
            long long a = wa[lane], bb = wb[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long ya = __shfl_up_sync(0xffffffffu, a, o), yb = __shfl_up_sync(0xffffffffu, bb, o);
                if (lane >= o) {
                    a += ya;
                    bb += yb;
                }
            }
            wa[lane] = a;
            wb[lane] = bb;
        }
        __syncthreads();
        const long long pa = ca + (warp ? wa[warp - 1] : 0) + xa - v.x;
        const long long pb = cb + (warp ? wb[warp - 1] : 0) + xb - v.y;
        // ids fit int32: the host rejects totals beyond that before the emit pass reads them
        if (s < n) bpre[s] = make_int2((int)(pa < 0x7fffffffll ? pa : 0x7fffffffll),
                                       (int)(pb < 0x7fffffffll ? pb : 0x7fffffffll));
        ca += wa[31];
        cb += wb[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        out[0] = ca;
        out[1] = cb;
    }
}

__global__ void __launch_bounds__(MC_T) mc_emit_kernel(const float* __restrict__ f, int R,
                                                       const uint64_t* __restrict__ chg,
                                                       const int32_t* __restrict__ n_slots,
                                                       const int32_t* __restrict__ slot_block,
                                                       const int32_t* __restrict__ block_slot,
                                                       const uint16_t* __restrict__ vloc,
                                                       const int2* __restrict__ bpre,
                                                       float* __restrict__ verts, int32_t* __restrict__ tris) {
    __shared__ int2 tmp[MC_T / 32];
    const int n = *n_slots;
    const int nb8 = R >> 3;
    for (int slot = blockIdx.x; slot < n; slot += gridDim.x) {   // uniform across the CTA
    const int b = slot_block[slot];
    const int bi = b / (nb8 * nb8), bj = (b / nb8) % nb8, bk = b % nb8;
    const bool band = block_band(chg, R, bi, bj, bk);
    const int l = threadIdx.x;
    const int i = 8 * bi + (l >> 6), j = 8 * bj + ((l >> 3) & 7), k = 8 * bk + (l & 7);
    const size_t s = ((size_t)i * R + j) * R + k;
    const float f0 = f[s];
    const float h = 2.0f / (float)R;
    // ---- this sample's vertices
    {
        int vid = bpre[slot].x + vloc[(size_t)slot * MC_T + l];
        const int idx[3] = {i, j, k};
        const size_t step[3] = {(size_t)R * R, (size_t)R, 1};
        for (int a = 0; a < 3; ++a) {
            if (idx[a] + 1 >= R) continue;
            const float f1 = f[s + step[a]];
            if ((f1 < 0.f) == (f0 < 0.f)) continue;
            const float t = f0 / (f0 - f1);
            float p[3] = {grid_coord(i, R), grid_coord(j, R), grid_coord(k, R)};
            p[a] += t * h;
            verts[(size_t)vid * 3] = p[0];
            verts[(size_t)vid * 3 + 1] = p[1];
            verts[(size_t)vid * 3 + 2] = p[2];
            ++vid;
        }
    }
    // ---- this cube's triangles
    const bool cube = band && i + 1 < R && j + 1 < R && k + 1 < R;
    const int cfg = cube ? cube_config(f, R, i, j, k) : 0;
    const int nt = cube ? c_mc.ntri[cfg] : 0;
    int2 tot;
    const int2 ex = mc_scan2(make_int2(nt, 0), tmp, tot);
    int tid = bpre[slot].y + ex.x;
    for (int q = 0; q < nt; ++q, ++tid) {
        for (int m = 0; m < 3; ++m) {
            const int e = c_mc.tri[cfg][q][m];
            const int a = e >> 2, u = (e >> 1) & 1, v = e & 1;
            // start corner of the edge: the owner sample
            int o[3] = {i, j, k};
            const int oth0 = a == 0 ? 1 : 0, oth1 = a == 2 ? 1 : 2;
            o[oth0] += u;
            o[oth1] += v;
            const int ob = ((o[0] >> 3) * nb8 + (o[1] >> 3)) * nb8 + (o[2] >> 3);
            const int os = min(block_slot[ob], n - 1);   // owner blocks are always visited
            const int ol = ((o[0] & 7) << 6) | ((o[1] & 7) << 3) | (o[2] & 7);
            const float fo = f[((size_t)o[0] * R + o[1]) * R + o[2]];
            const int rank = own_edges(f, R, o[0], o[1], o[2], a, fo);
            tris[(size_t)tid * 3 + m] = bpre[os].x + vloc[(size_t)os * MC_T + ol] + rank;
        }
    }
    }
}

std::mutex g_mc_mu;
bool g_mc_ok = false, g_mc_built = false;
McTable g_mc_host;
constexpr int kMaxDev = 64;
bool g_mc_uploaded[kMaxDev] = {};

struct McPlan {
    size_t off_bits, off_chg, off_flag, off_word_off, off_ids, off_toff, off_counts, off_tmp, off_vloc, off_btot,
        off_bpre, off_out, total;
};

McPlan mc_plan(int R) {
    McPlan p;
    const size_t nw = (size_t)(R / 4) * (R / 4) * (R / 4);
    const size_t nb = (size_t)(R / 8) * (R / 8) * (R / 8);
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t o = 0;
    p.off_bits = o;     o = up(o + 2 * nw * 8);
    p.off_chg = o;      o = up(o + nw * 8);
    p.off_flag = o;     o = up(o + nb * 8);
    p.off_word_off = o; o = up(o + (nb + 1) * 4);
    p.off_ids = o;      o = up(o + nb * 4);
    p.off_toff = o;     o = up(o + (nb + 1) * 4);
    p.off_counts = o;   o = up(o + 16);
    p.off_tmp = o;      o = up(o + compact_tmp_ints((int)nb) * 4);
    p.off_vloc = o;     o = up(o + nb * MC_T * 2);
    p.off_btot = o;     o = up(o + nb * 8);
    p.off_bpre = o;     o = up(o + nb * 8);
    p.off_out = o;      o = up(o + 16);
    p.total = o + 256;
    return p;
}

}  // namespace
}  // namespace vdm

using namespace vdm;

extern "C" {

vdm_status vdm_surface_case_table(uint8_t* ntri, uint8_t* tri) {
    if (!ntri || !tri) return fail(VDM_ERR_INVALID_ARG, "null output");
    std::lock_guard<std::mutex> lock(g_mc_mu);
    if (!g_mc_built) {
        g_mc_ok = build_table(g_mc_host);
        g_mc_built = true;
    }
    if (!g_mc_ok) return fail(VDM_ERR_INTERNAL, "marching cubes case table could not be built");
    memcpy(ntri, g_mc_host.ntri, 256);
    memcpy(tri, g_mc_host.tri, sizeof(g_mc_host.tri));
    return VDM_OK;
}

vdm_status vdm_surface_workspace_size(int32_t R, size_t* bytes) {
    if (!bytes) return fail(VDM_ERR_INVALID_ARG, "bytes is NULL");
    if (R < 8 || R % 8 || R > 1024) return fail(VDM_ERR_UNSUPPORTED, "R = %d must be a multiple of 8 in [8, 1024]", R);
    *bytes = mc_plan(R).total;
    return VDM_OK;
}

vdm_status vdm_extract_surface(const float* d_f, int32_t R, float* d_vertices, int64_t max_vertices,
                               int32_t* d_triangles, int64_t max_triangles, int64_t* n_vertices,
                               int64_t* n_triangles, void* d_ws, size_t ws_bytes, vdm_stream stream) {
    size_t need = 0;
    VDM_TRY(vdm_surface_workspace_size(R, &need));
    if (!d_f || !n_vertices || !n_triangles) return fail(VDM_ERR_INVALID_ARG, "null f / counts");
    if (max_vertices < 0 || max_triangles < 0) return fail(VDM_ERR_INVALID_ARG, "negative capacity");
    if ((max_vertices > 0 && !d_vertices) || (max_triangles > 0 && !d_triangles))
        return fail(VDM_ERR_INVALID_ARG, "null vertex / triangle buffer with a non-zero capacity");
    if ((uintptr_t)d_f % 16) return fail(VDM_ERR_INVALID_ARG, "f must be 16-byte aligned");
    if (!d_ws || ws_bytes < need) return fail(VDM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    void* ws = reinterpret_cast<void*>(((uintptr_t)d_ws + 255) & ~(uintptr_t)255);
    if ((uintptr_t)ws - (uintptr_t)d_ws + need - 256 > ws_bytes)
        return fail(VDM_ERR_WORKSPACE, "workspace too small after alignment");
    int dev = 0;
    VDM_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDev) return fail(VDM_ERR_UNSUPPORTED, "device %d out of range", dev);
    {
        std::lock_guard<std::mutex> lock(g_mc_mu);
        if (!g_mc_built) {
            g_mc_ok = build_table(g_mc_host);
            g_mc_built = true;
        }
        if (!g_mc_ok) return fail(VDM_ERR_INTERNAL, "marching cubes case table could not be built");
        if (!g_mc_uploaded[dev]) {
            VDM_CUDA_TRY(cudaMemcpyToSymbol(c_mc, &g_mc_host, sizeof(McTable)));
            g_mc_uploaded[dev] = true;
        }
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const McPlan pl = mc_plan(R);
    char* w = static_cast<char*>(ws);
    uint64_t* bits = reinterpret_cast<uint64_t*>(w + pl.off_bits);
    uint64_t* chg = reinterpret_cast<uint64_t*>(w + pl.off_chg);
    uint64_t* flag = reinterpret_cast<uint64_t*>(w + pl.off_flag);
    int32_t* word_off = reinterpret_cast<int32_t*>(w + pl.off_word_off);
    int32_t* ids = reinterpret_cast<int32_t*>(w + pl.off_ids);
    int32_t* toff = reinterpret_cast<int32_t*>(w + pl.off_toff);
    int32_t* counts = reinterpret_cast<int32_t*>(w + pl.off_counts);
    int32_t* tmp = reinterpret_cast<int32_t*>(w + pl.off_tmp);
    uint16_t* vloc = reinterpret_cast<uint16_t*>(w + pl.off_vloc);
    int2* btot = reinterpret_cast<int2*>(w + pl.off_btot);
    int2* bpre = reinterpret_cast<int2*>(w + pl.off_bpre);
    long long* out = reinterpret_cast<long long*>(w + pl.off_out);
    const int nb8 = R / 8;
    const int nblk = nb8 * nb8 * nb8;
    VDM_TRY(launch_sign_change(d_f, R, chg, bits, st));
    mc_flag_kernel<<<(nblk + 255) / 256, 256, 0, st>>>(chg, R, flag);
    VDM_TRY(check_launch("mc_flag_kernel"));
    // flagged blocks -> slot list (ids) and block -> slot map (word_off), no parent list
    VDM_TRY(launch_compact(flag, nblk, R, word_off, ids, toff, nullptr, counts, tmp, st));
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = nblk < sms * 4 ? nblk : sms * 4;   // persistent CTAs over the flagged blocks
    mc_count_kernel<<<grid, MC_T, 0, st>>>(d_f, R, chg, counts + 1, ids, vloc, btot);
    VDM_TRY(check_launch("mc_count_kernel"));
    mc_scan_kernel<<<1, 1024, 0, st>>>(btot, counts + 1, bpre, out);
    VDM_TRY(check_launch("mc_scan_kernel"));
    long long hc[2] = {0, 0};
    VDM_CUDA_TRY(cudaMemcpyAsync(hc, out, sizeof(hc), cudaMemcpyDeviceToHost, st));
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    *n_vertices = hc[0];
    *n_triangles = hc[1];
    if (hc[0] > 0x7fffffffll || hc[1] > 0x7fffffffll)
        return fail(VDM_ERR_UNSUPPORTED, "mesh of %lld vertices / %lld triangles exceeds int32 ids", hc[0], hc[1]);
    if (hc[0] > max_vertices || hc[1] > max_triangles)
        return fail(VDM_ERR_WORKSPACE, "mesh needs %lld vertices and %lld triangles (capacity %lld, %lld)", hc[0],
                    hc[1], (long long)max_vertices, (long long)max_triangles);
    if (hc[0] == 0 && hc[1] == 0) return VDM_OK;
    mc_emit_kernel<<<grid, MC_T, 0, st>>>(d_f, R, chg, counts + 1, ids, word_off, vloc, bpre, d_vertices, d_triangles);
    VDM_TRY(check_launch("mc_emit_kernel"));
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    return VDM_OK;
}

}  // extern "C"
