// Host side of the C ABI declared in include/vdm.h: argument checks, workspace
// planning, the coarse-to-fine level driver and kernel launches.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "vdm_internal.cuh"

namespace vdm {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

vdm_status fail(vdm_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

vdm_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return VDM_OK;
}

int decode_simt_chunk();

namespace {

size_t elt_size(vdm_dtype d) { return d == VDM_F32 ? 4 : 2; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

vdm_status check_decoder(const vdm_decoder* d, bool need_query_side) {
    if (!d) return fail(VDM_ERR_INVALID_ARG, "decoder is NULL");
    if (d->dtype != VDM_F32 && d->dtype != VDM_BF16)
        return fail(VDM_ERR_INVALID_ARG, "unknown dtype %d", (int)d->dtype);
    if (d->H < 1 || d->C != d->H * kHeadDim)
        return fail(VDM_ERR_UNSUPPORTED, "C (%d) must equal 64 * H (H = %d)", d->C, d->H);
    if (d->C != 64 && d->C != 128 && d->C != 256 && d->C != 512)
        return fail(VDM_ERR_UNSUPPORTED, "C = %d not in {64, 128, 256, 512}", d->C);
    if (d->F < 64 || d->F > 4096 || d->F % 64)
        return fail(VDM_ERR_UNSUPPORTED, "F = %d must be a multiple of 64 in [64, 4096]", d->F);
    if (d->query_ln != 0 && d->query_ln != 1)
        return fail(VDM_ERR_INVALID_ARG, "query_ln must be 0 or 1");
    const size_t al = 16;
    const void* mats[] = {d->Wq, d->Wk, d->Wv, d->Wo, d->W1, d->W2};
    const char* names[] = {"Wq", "Wk", "Wv", "Wo", "W1", "W2"};
    for (int i = 0; i < 6; ++i) {
        if (!need_query_side && i != 1 && i != 2) continue;
        if (!mats[i]) return fail(VDM_ERR_INVALID_ARG, "%s is NULL", names[i]);
        if (!aligned(mats[i], al)) return fail(VDM_ERR_INVALID_ARG, "%s is not %zu-byte aligned", names[i], al);
    }
    const float* vecs[] = {d->bk, d->bv, d->ln_kv_g, d->ln_kv_b, d->bq, d->bo, d->b1, d->b2,
                           d->ln1_g, d->ln1_b, d->ln2_g, d->ln2_b, d->w_head, d->b_head};
    const int nvec = need_query_side ? 14 : 4;
    for (int i = 0; i < nvec; ++i) {
        if (!vecs[i]) return fail(VDM_ERR_INVALID_ARG, "decoder vector %d is NULL", i);
        if (i < 13 && !aligned(vecs[i], 16))
            return fail(VDM_ERR_INVALID_ARG, "decoder vector %d is not 16-byte aligned", i);
    }
    if (need_query_side && d->w_tsdf) {
        if (!d->b_tsdf) return fail(VDM_ERR_INVALID_ARG, "tSDF head: b_tsdf is NULL");
        if (!aligned(d->w_tsdf, 16)) return fail(VDM_ERR_INVALID_ARG, "w_tsdf is not 16-byte aligned");
    }
    return VDM_OK;
}

vdm_status check_analytic(const vdm_decoder* d, const vdm_analytic* an) {
    if (!an) return VDM_OK;
    if (!an->spheres || an->n_spheres < 1)
        return fail(VDM_ERR_INVALID_ARG, "analytic term needs spheres and n_spheres >= 1");
    if (d->w_tsdf && !(an->tsdf_trunc > 0.f))
        return fail(VDM_ERR_INVALID_ARG, "a tSDF head with an analytic term needs tsdf_trunc > 0");
    return VDM_OK;
}

DecodeArgs base_args(const vdm_decoder* d, const void* K, const void* V, int N) {
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.C = d->C; a.H = d->H; a.F = d->F; a.query_ln = d->query_ln;
    a.Wq = d->Wq; a.Wo = d->Wo; a.W1 = d->W1; a.W2 = d->W2;
    a.bq = d->bq; a.bo = d->bo; a.b1 = d->b1; a.b2 = d->b2;
    a.ln1_g = d->ln1_g; a.ln1_b = d->ln1_b; a.ln2_g = d->ln2_g; a.ln2_b = d->ln2_b;
    a.w_head = d->w_head; a.b_head = d->b_head;
    a.w_tsdf = d->w_tsdf; a.b_tsdf = d->b_tsdf;
    a.K = K; a.V = V; a.N = N;
    return a;
}

size_t kv_shape_bytes(const vdm_decoder* d, int N) {
    return (size_t)d->H * N * kHeadDim * elt_size(d->dtype);
}

// ---------------------------------------------------------------- workspace plan
struct Plan {
    int L;
    int R[VDM_MAX_LEVELS];
    size_t off_grid[VDM_MAX_LEVELS];
    size_t off_tgrid[VDM_MAX_LEVELS];   // tSDF grids of levels 0 .. L-2 (decoders with a tSDF head)
    size_t off_words, off_bits, off_word_off, off_tile_ids, off_tile_off, off_counts, off_scan, off_plist,
        off_qorder, off_sel, off_seltiles, off_ml, off_dense, off_dense_ml, off_units, off_units_n;
    int nw_max;
    int k;
    size_t ml_bytes;
    size_t total;
};

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

vdm_status make_plan(const vdm_hier_params* p, int N, int ml_heads, bool tsdf, Plan& pl) {
    if (!p) return fail(VDM_ERR_INVALID_ARG, "params is NULL");
    if (p->n_levels < 1 || p->n_levels > VDM_MAX_LEVELS)
        return fail(VDM_ERR_UNSUPPORTED, "n_levels = %d not in [1, %d]", p->n_levels, VDM_MAX_LEVELS);
    if (p->r0 < 4 || p->r0 % 4) return fail(VDM_ERR_UNSUPPORTED, "r0 = %d must be a positive multiple of 4", p->r0);
    const int64_t rf = (int64_t)p->r0 << (p->n_levels - 1);
    if (rf > 1024) return fail(VDM_ERR_UNSUPPORTED, "final resolution %lld > 1024", (long long)rf);
    if (p->adaptive) {
        if (p->tile != 8) return fail(VDM_ERR_UNSUPPORTED, "sub-volume edge must be 8 (got %d)", p->tile);
        if (p->n_probe < 1 || p->n_probe > 512) return fail(VDM_ERR_UNSUPPORTED, "n_probe must be in [1, 512]");
        if (p->top_k < 1) return fail(VDM_ERR_INVALID_ARG, "top_k must be >= 1");
    }
    if (tsdf && !(p->tsdf_threshold > 0.f))
        return fail(VDM_ERR_INVALID_ARG, "a tSDF head needs tsdf_threshold > 0");
    pl.L = p->n_levels;
    pl.k = p->adaptive ? (p->top_k < N ? p->top_k : N) : 0;
    size_t o = 0;
    int nw_max = 0;
    int64_t vox_max = 0;
    for (int l = 0; l < pl.L; ++l) {
        pl.R[l] = p->r0 << l;
        if (l < pl.L - 1) {
            pl.off_grid[l] = o;
            o = align_up(o + (size_t)pl.R[l] * pl.R[l] * pl.R[l] * 4);
            pl.off_tgrid[l] = o;
            if (tsdf) o = align_up(o + (size_t)pl.R[l] * pl.R[l] * pl.R[l] * 4);
            const int nb = pl.R[l] / 4;
            if (nb * nb * nb > nw_max) nw_max = nb * nb * nb;
            const int64_t v = (int64_t)pl.R[l] * pl.R[l] * pl.R[l];
            if (v > vox_max) vox_max = v;
        }
    }
    pl.nw_max = nw_max;
    pl.off_words = o;     o = align_up(o + (size_t)nw_max * 8);
    pl.off_bits = o;      o = align_up(o + (size_t)nw_max * 2 * 8);
    pl.off_word_off = o;  o = align_up(o + (size_t)(nw_max + 1) * 4);
    pl.off_tile_ids = o;  o = align_up(o + (size_t)nw_max * 4);
    pl.off_tile_off = o;  o = align_up(o + (size_t)(nw_max + 1) * 4);
    pl.off_counts = o;    o = align_up(o + 4 * 4 * VDM_MAX_LEVELS);
    pl.off_scan = o;      o = align_up(o + compact_tmp_ints(nw_max) * 4);
    pl.off_plist = o;     o = align_up(o + (size_t)vox_max * 4);
    pl.off_qorder = o;    o = align_up(o + (p->adaptive ? (size_t)vox_max * 8 * 4 : 0));
    pl.off_sel = o;       o = align_up(o + (p->adaptive ? (size_t)nw_max * pl.k * 4 : 0));
    pl.off_seltiles = o;  o = align_up(o + (p->adaptive ? (size_t)nw_max * 4 : 0));
    pl.ml_bytes = p->adaptive ? (size_t)nw_max * p->n_probe * ml_heads * 2 * 4 : 0;
    pl.off_ml = o;        o = align_up(o + pl.ml_bytes);
    const size_t dense_max = p->adaptive ? (size_t)nw_max * (p->n_probe < 512 ? p->n_probe : 512) : 0;
    pl.off_dense = o;     o = align_up(o + dense_max * 4);
    pl.off_dense_ml = o;  o = align_up(o + dense_max * 4);
    // the sparse pass's non-empty (sub-volume, slot) units: at most 512 / 128 slots per sub-volume
    pl.off_units = o;     o = align_up(o + (p->adaptive ? (size_t)nw_max * 4 * 4 : 0));
    pl.off_units_n = o;   o = align_up(o + 4);
    pl.total = o + 256;
    return VDM_OK;
}

template <typename T> T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace
}  // namespace vdm

using namespace vdm;

extern "C" {

int32_t vdm_abi_version(void) { return 3; }

const char* vdm_last_error(void) { return g_err; }

const char* vdm_status_string(vdm_status s) {
    switch (s) {
        case VDM_OK: return "ok";
        case VDM_ERR_INVALID_ARG: return "invalid argument";
        case VDM_ERR_UNSUPPORTED: return "unsupported shape";
        case VDM_ERR_WORKSPACE: return "workspace too small";
        case VDM_ERR_CUDA: return "CUDA error";
        case VDM_ERR_TIMEOUT: return "device wait timed out";
        case VDM_ERR_INTERNAL: return "internal error";
    }
    return "unknown status";
}

vdm_status vdm_precompute_kv(const vdm_decoder* dec, const float* d_z, int32_t B, int32_t N,
                             void* d_k_out, void* d_v_out, vdm_stream stream) {
    VDM_TRY(check_decoder(dec, false));
    if (B < 1 || N < 1) return fail(VDM_ERR_INVALID_ARG, "B and N must be >= 1");
    if (N > kMaxN) return fail(VDM_ERR_UNSUPPORTED, "N = %d > %d", N, kMaxN);
    if (!d_z || !d_k_out || !d_v_out) return fail(VDM_ERR_INVALID_ARG, "null z / k / v");
    if (!aligned(d_k_out, 16) || !aligned(d_v_out, 16))
        return fail(VDM_ERR_INVALID_ARG, "k / v must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t kvb = kv_shape_bytes(dec, N);
    for (int b = 0; b < B; ++b) {
        KvArgs a;
        a.C = dec->C; a.H = dec->H; a.N = N;
        a.z = d_z + (size_t)b * N * dec->C;
        a.Wk = dec->Wk; a.Wv = dec->Wv; a.bk = dec->bk; a.bv = dec->bv;
        a.g = dec->ln_kv_g; a.b = dec->ln_kv_b;
        a.K = static_cast<char*>(d_k_out) + b * kvb;
        a.V = static_cast<char*>(d_v_out) + b * kvb;
        VDM_TRY(launch_precompute_kv(a, dec->dtype, st));
    }
    return VDM_OK;
}

vdm_status vdm_decode_dense(const vdm_decoder* dec, const void* d_k, const void* d_v, int32_t B,
                            int32_t N, const float* d_xyz, int64_t M, int32_t grid_R,
                            const vdm_analytic* an, float* d_out, vdm_stream stream) {
    VDM_TRY(check_decoder(dec, true));
    if (B < 1 || N < 1 || M < 0) return fail(VDM_ERR_INVALID_ARG, "B, N must be >= 1 and M >= 0");
    if (N > kMaxN) return fail(VDM_ERR_UNSUPPORTED, "N = %d > %d", N, kMaxN);
    if (M == 0) return VDM_OK;
    if (!d_k || !d_v || !d_out) return fail(VDM_ERR_INVALID_ARG, "null k / v / out");
    if (!d_xyz) {
        if (grid_R < 1 || (int64_t)grid_R * grid_R * grid_R != M)
            return fail(VDM_ERR_INVALID_ARG, "grid mode needs M == grid_R^3 (M = %lld, R = %d)",
                        (long long)M, grid_R);
    }
    if (M > ((int64_t)1 << 31) - 1) return fail(VDM_ERR_UNSUPPORTED, "M too large");
    VDM_TRY(check_analytic(dec, an));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t kvb = kv_shape_bytes(dec, N);
    for (int b = 0; b < B; ++b) {
        DecodeArgs a = base_args(dec, static_cast<const char*>(d_k) + b * kvb,
                                 static_cast<const char*>(d_v) + b * kvb, N);
        a.work = kWorkFlat;
        a.M = M;
        if (d_xyz) {
            a.qmode = kQueryXyz;
            a.xyz = d_xyz + (size_t)b * M * 3;
        } else {
            a.qmode = kQueryGrid;
            a.R = grid_R;
        }
        a.out = d_out + (size_t)b * M;
        if (an) {
            a.spheres = an->spheres + (size_t)b * an->n_spheres * 4;
            a.n_spheres = an->n_spheres;
            a.dec_scale = an->dec_scale;
            a.tsdf_trunc = an->tsdf_trunc;
        }
        VDM_TRY(launch_decode(a, dec->dtype, st));
    }
    // the status of the kernels' bounded waits reaches the caller who made this call
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    return tc_check_error();
}

vdm_status vdm_select_kv(const vdm_decoder* dec, const void* d_k, const void* d_v, int32_t N,
                         const float* d_probe_xyz, const int32_t* d_tile_off, int32_t T,
                         int64_t P_total, int32_t top_k, int32_t* d_sel_out, float* d_score_out,
                         float* d_probe_dec_out, vdm_stream stream) {
    VDM_TRY(check_decoder(dec, true));
    if (N < 1 || T < 0 || P_total < 0) return fail(VDM_ERR_INVALID_ARG, "bad N / T / P");
    if (N > kMaxN) return fail(VDM_ERR_UNSUPPORTED, "N = %d > %d", N, kMaxN);
    if (top_k < 1 || top_k > N) return fail(VDM_ERR_INVALID_ARG, "top_k must be in [1, N]");
    if (T == 0) return VDM_OK;
    if (!d_k || !d_v || !d_tile_off || !d_sel_out || (P_total > 0 && !d_probe_xyz))
        return fail(VDM_ERR_INVALID_ARG, "null k / v / tile_off / sel / probe_xyz");
    if (P_total > ((int64_t)1 << 31) - 1) return fail(VDM_ERR_UNSUPPORTED, "P too large");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the offsets are checked on the host; the largest probe count picks the probe rows per sub-volume
    std::vector<int32_t> off((size_t)T + 1);
    VDM_CUDA_TRY(cudaMemcpyAsync(off.data(), d_tile_off, ((size_t)T + 1) * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    if (off[0] != 0 || (int64_t)off[T] != P_total)
        return fail(VDM_ERR_INVALID_ARG, "tile_off[0] must be 0 and tile_off[T] = P (%lld, got %d .. %d)",
                    (long long)P_total, off[0], off[T]);
    int max_count = 0;
    for (int t = 0; t < T; ++t) {
        const int c = off[t + 1] - off[t];
        if (c < 0) return fail(VDM_ERR_INVALID_ARG, "tile_off must be non-decreasing (tile %d)", t);
        max_count = std::max(max_count, c);
    }
    // Tensor-core route, the kernels of the hierarchical path: the probes are decoded with full
    // attention (exporting their per-head softmax maximum and sum), then scored in one pass
    DecodeArgs d = base_args(dec, d_k, d_v, N);
    d.work = kWorkFlat;
    d.qmode = kQueryXyz;
    d.xyz = d_probe_xyz;
    d.M = P_total;
    int np = 0;
    for (int c : {32, 64, 128})
        if (np == 0 && max_count <= c && select_tc_supported(dec->C, c, N, dec->dtype)) np = c;
    if (P_total > 0 && np > 0 && tc_supported(d, dec->dtype)) {
        size_t o = 0;
        const size_t o_ml = o;
        o = align_up(o + (size_t)T * np * dec->H * 2 * sizeof(float));
        const size_t o_slot = o;
        o = align_up(o + (size_t)P_total * sizeof(int32_t));
        const size_t o_tiles = o;
        o = align_up(o + (size_t)T * sizeof(int32_t));
        const size_t o_n = o;
        o = align_up(o + sizeof(int32_t));
        void* tmp = nullptr;
        VDM_CUDA_TRY(cudaMallocAsync(&tmp, o, st));
        auto run = [&]() -> vdm_status {
            float* probe_ml = at<float>(tmp, o_ml);
            int32_t* ml_slot = at<int32_t>(tmp, o_slot);
            int32_t* sel_tiles = at<int32_t>(tmp, o_tiles);
            int32_t* n_sel = at<int32_t>(tmp, o_n);
            VDM_TRY(launch_flat_probe_slots(d_tile_off, T, np, ml_slot, sel_tiles, n_sel, st));
            d.probe_ml = probe_ml;
            d.ml_slot = ml_slot;
            d.out = d_probe_dec_out;   // the probes' decoded values, when asked for
            VDM_TRY(launch_decode_tc(d, st));
            SelectTcLaunch L{};
            L.C = dec->C; L.H = dec->H; L.N = N;
            L.Wq = dec->Wq; L.bq = dec->bq; L.K = d_k;
            L.T = T;
            L.n_sel = n_sel;
            L.sel_tiles = sel_tiles;
            L.probe_xyz = d_probe_xyz;
            L.probe_off = d_tile_off;
            L.probe_ml = probe_ml;
            L.n_probe = np;
            L.top_k = top_k;
            L.sel = d_sel_out;
            L.score_out = d_score_out;
            L.score_rows = d_score_out ? T : 0;
            return launch_select_tc(L, st);
        };
        const vdm_status r = run();
        const cudaError_t fe = cudaFreeAsync(tmp, st);
        VDM_TRY(r);
        if (fe != cudaSuccess) return fail(VDM_ERR_CUDA, "cudaFreeAsync: %s", cudaGetErrorString(fe));
    } else {
        // CUDA-core route: any dtype, width and probe count
        SelectArgs a;
        memset(&a, 0, sizeof(a));
        a.C = dec->C; a.H = dec->H; a.N = N;
        a.Wq = dec->Wq; a.bq = dec->bq; a.K = d_k;
        a.T = T;
        a.probe_xyz = d_probe_xyz ? d_probe_xyz : reinterpret_cast<const float*>(d_tile_off);
        a.probe_off = d_tile_off;
        a.top_k = top_k;
        a.sel = d_sel_out;
        a.score = d_score_out;
        VDM_TRY(launch_select(a, dec->dtype, st));
        if (d_probe_dec_out && P_total > 0) {
            d.out = d_probe_dec_out;
            VDM_TRY(launch_decode(d, dec->dtype, st));
        }
    }
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    return tc_check_error();
}

// encoder workspace: point features u [M][C] fp32, keys and values [H][M][64] in the block's dtype
static size_t encode_ws_bytes(const vdm_decoder* blk, int M, size_t* off) {
    size_t o = 0;
    off[0] = o; o = align_up(o + (size_t)M * blk->C * 4);
    off[1] = o; o = align_up(o + kv_shape_bytes(blk, M));
    off[2] = o; o = align_up(o + kv_shape_bytes(blk, M));
    return o + 256;
}

vdm_status vdm_encode_workspace_size(const vdm_decoder* blk, int32_t M, size_t* bytes) {
    VDM_TRY(check_decoder(blk, true));
    if (!bytes) return fail(VDM_ERR_INVALID_ARG, "bytes is NULL");
    if (M < 1 || M > kMaxN) return fail(VDM_ERR_UNSUPPORTED, "M = %d not in [1, %d]", M, kMaxN);
    size_t off[3];
    *bytes = encode_ws_bytes(blk, M, off);
    return VDM_OK;
}

vdm_status vdm_encode(const vdm_decoder* blk, const void* d_W_in, const float* d_b_in, const float* d_points,
                      int32_t B, int32_t M, const float* d_queries, int32_t N, float* d_z_out, void* d_ws,
                      size_t ws_bytes, vdm_stream stream) {
    size_t need = 0;
    VDM_TRY(vdm_encode_workspace_size(blk, M, &need));
    if (B < 1 || N < 1) return fail(VDM_ERR_INVALID_ARG, "B and N must be >= 1");
    if (!d_W_in || !d_b_in || !d_points || !d_queries || !d_z_out)
        return fail(VDM_ERR_INVALID_ARG, "null W_in / b_in / points / queries / z_out");
    if (!aligned(d_W_in, 16) || !aligned(d_b_in, 16) || !aligned(d_z_out, 16))
        return fail(VDM_ERR_INVALID_ARG, "W_in, b_in and z_out must be 16-byte aligned");
    if (!d_ws || ws_bytes < need) return fail(VDM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    void* ws = reinterpret_cast<void*>(align_up((uintptr_t)d_ws));
    if ((uintptr_t)ws - (uintptr_t)d_ws + need - 256 > ws_bytes)
        return fail(VDM_ERR_WORKSPACE, "workspace too small after alignment");
    size_t off[3];
    encode_ws_bytes(blk, M, off);
    float* u = at<float>(ws, off[0]);
    void* K = at<char>(ws, off[1]);
    void* V = at<char>(ws, off[2]);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int b = 0; b < B; ++b) {
        // keys and values from the cloud: embedded, projected, LayerNormed points
        VDM_TRY(launch_point_features(d_points + (size_t)b * M * 3, M, blk->C, d_W_in, d_b_in, u, blk->dtype, st));
        KvArgs k;
        k.C = blk->C; k.H = blk->H; k.N = M;
        k.z = u;
        k.Wk = blk->Wk; k.Wv = blk->Wv; k.bk = blk->bk; k.bv = blk->bv;
        k.g = blk->ln_kv_g; k.b = blk->ln_kv_b;
        k.K = K; k.V = V;
        VDM_TRY(launch_precompute_kv(k, blk->dtype, st));
        // the latent tokens run the block from their query points; the output is the block's x2
        DecodeArgs a = base_args(blk, K, V, M);
        a.w_tsdf = nullptr;
        a.work = kWorkFlat;
        a.qmode = kQueryXyz;
        a.xyz = d_queries + (size_t)b * N * 3;
        a.M = N;
        a.feat_out = d_z_out + (size_t)b * N * blk->C;
        VDM_TRY(launch_decode(a, blk->dtype, st));
    }
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    return tc_check_error();
}

static size_t refine_ws_bytes(int R, size_t* off) {
    const size_t nw = (size_t)(R / 4) * (R / 4) * (R / 4);
    size_t o = 0;
    off[0] = o; o = align_up(o + mark_bits_words(R) * 8);         // sign / near words
    off[1] = o; o = align_up(o + (nw + 1) * 4);                   // word offsets
    off[2] = o; o = align_up(o + nw * 4);                         // non-empty word ids
    off[3] = o; o = align_up(o + (nw + 1) * 4);                   // their parent offsets
    off[4] = o; o = align_up(o + compact_tmp_ints((int)nw) * 4);  // chunk sums
    return o + 256;
}

vdm_status vdm_refine_workspace_size(int32_t R, size_t* bytes) {
    if (!bytes) return fail(VDM_ERR_INVALID_ARG, "bytes is NULL");
    if (R < 4 || R % 4 || R > 512) return fail(VDM_ERR_UNSUPPORTED, "R = %d must be a multiple of 4 in [4, 512]", R);
    size_t off[5];
    *bytes = refine_ws_bytes(R, off);
    return VDM_OK;
}

vdm_status vdm_refine_level(const float* d_f, int32_t R, float* d_f_fine, uint64_t* d_mask, int32_t* d_parents,
                            int32_t* d_counts, void* d_ws, size_t ws_bytes, vdm_stream stream) {
    size_t need = 0;
    VDM_TRY(vdm_refine_workspace_size(R, &need));
    if (!d_f || !d_mask || !d_counts) return fail(VDM_ERR_INVALID_ARG, "null f / mask / counts");
    if ((uintptr_t)d_f % 16 || (d_f_fine && (uintptr_t)d_f_fine % 16))
        return fail(VDM_ERR_INVALID_ARG, "grids must be 16-byte aligned");
    if (!d_ws || ws_bytes < need) return fail(VDM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    void* ws = reinterpret_cast<void*>(align_up((uintptr_t)d_ws));
    if ((uintptr_t)ws - (uintptr_t)d_ws + need - 256 > ws_bytes)
        return fail(VDM_ERR_WORKSPACE, "workspace too small after alignment");
    size_t off[5];
    refine_ws_bytes(R, off);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int nw = (R / 4) * (R / 4) * (R / 4);
    VDM_TRY(launch_mark_dilate(d_f, d_f, R, (float)(4.0 / (double)R), d_mask, at<uint64_t>(ws, off[0]), st));
    VDM_TRY(launch_compact(d_mask, nw, R, at<int32_t>(ws, off[1]), at<int32_t>(ws, off[2]), at<int32_t>(ws, off[3]),
                           d_parents, d_counts, at<int32_t>(ws, off[4]), st));
    if (d_f_fine) VDM_TRY(launch_fill(d_f, R, d_f_fine, st));
    return VDM_OK;
}

vdm_status vdm_hierarchical_workspace_size(const vdm_decoder* dec, const vdm_hier_params* p, int32_t N,
                                           size_t* bytes) {
    VDM_TRY(check_decoder(dec, true));
    if (!bytes) return fail(VDM_ERR_INVALID_ARG, "bytes is NULL");
    if (N < 1 || N > kMaxN) return fail(VDM_ERR_UNSUPPORTED, "N = %d not in [1, %d]", N, kMaxN);
    Plan pl;
    VDM_TRY(make_plan(p, N, dec->H, dec->w_tsdf != nullptr, pl));
    *bytes = pl.total;
    return VDM_OK;
}

vdm_status vdm_decode_hierarchical(const vdm_decoder* dec, const void* d_k, const void* d_v,
                                   int32_t B, int32_t N, const vdm_hier_params* p,
                                   const vdm_analytic* an, float* d_grid_out, void* d_ws,
                                   size_t ws_bytes, vdm_hier_stats* stats, const vdm_hier_debug* dbg,
                                   vdm_stream stream) {
    VDM_TRY(check_decoder(dec, true));
    if (B < 1 || N < 1) return fail(VDM_ERR_INVALID_ARG, "B and N must be >= 1");
    if (N > kMaxN) return fail(VDM_ERR_UNSUPPORTED, "N = %d > %d", N, kMaxN);
    if (!d_k || !d_v || !d_grid_out) return fail(VDM_ERR_INVALID_ARG, "null k / v / grid_out");
    VDM_TRY(check_analytic(dec, an));
    const bool tsdf = dec->w_tsdf != nullptr;
    Plan pl;
    VDM_TRY(make_plan(p, N, dec->H, tsdf, pl));
    if (dbg) {
        bool any_attn = false;
        for (int l = 0; l < VDM_MAX_LEVELS; ++l) any_attn |= dbg->attn[l] != nullptr;
        if (any_attn && dbg->attn_stride < 1)
            return fail(VDM_ERR_INVALID_ARG, "debug attn needs attn_stride >= 1");
    }
    if (pl.L > 1 && (!d_ws || ws_bytes < pl.total))
        return fail(VDM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", pl.total, ws_bytes);
    void* ws = d_ws ? reinterpret_cast<void*>(align_up((uintptr_t)d_ws)) : nullptr;
    if (ws && (uintptr_t)ws - (uintptr_t)d_ws + pl.total - 256 > ws_bytes)
        return fail(VDM_ERR_WORKSPACE, "workspace too small after alignment");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t kvb = kv_shape_bytes(dec, N);
    const int L = pl.L;
    const int64_t Rf = pl.R[L - 1];

    for (int b = 0; b < B; ++b) {
        const void* K = static_cast<const char*>(d_k) + b * kvb;
        const void* V = static_cast<const char*>(d_v) + b * kvb;
        float* grid[VDM_MAX_LEVELS];
        for (int l = 0; l < L - 1; ++l) grid[l] = at<float>(ws, pl.off_grid[l]);
        grid[L - 1] = d_grid_out + (size_t)b * Rf * Rf * Rf;
        // tSDF grids: workspace for the marked levels, the caller's debug array (if any) at the last
        float* tgrid[VDM_MAX_LEVELS] = {};
        if (tsdf) {
            for (int l = 0; l < L - 1; ++l) tgrid[l] = at<float>(ws, pl.off_tgrid[l]);
            if (dbg && dbg->tsdf[L - 1]) tgrid[L - 1] = dbg->tsdf[L - 1] + (size_t)b * Rf * Rf * Rf;
        }
        DecodeArgs base = base_args(dec, K, V, N);
        if (an) {
            base.spheres = an->spheres + (size_t)b * an->n_spheres * 4;
            base.n_spheres = an->n_spheres;
            base.dec_scale = an->dec_scale;
            base.tsdf_trunc = an->tsdf_trunc;
        }
        vdm_hier_stats* sb = stats ? stats + b : nullptr;
        if (sb) memset(sb, 0, sizeof(*sb));
        auto dbg_ptr = [&](float* const* arr, int l, int64_t per) -> float* {
            return (dbg && arr[l]) ? arr[l] + (size_t)b * per : nullptr;
        };
        // attention-output rows of level l: one per attn_stride voxels
        auto attn_ptr = [&](int l) -> float* {
            if (!dbg || !dbg->attn[l]) return nullptr;
            const int64_t R = pl.R[l];
            const int64_t rows = (R * R * R + dbg->attn_stride - 1) / dbg->attn_stride;
            return dbg->attn[l] + (size_t)b * rows * dec->C;
        };
        const int64_t astride = dbg ? dbg->attn_stride : 0;
        // ---- level 0: dense
        {
            const int R = pl.R[0];
            DecodeArgs a = base;
            a.work = kWorkFlat;
            a.qmode = kQueryGrid;
            a.R = R;
            a.M = (int64_t)R * R * R;
            a.grid = grid[0];
            a.tsdf_grid = tgrid[0];
            a.dec_grid = dbg_ptr(dbg ? dbg->dec : nullptr, 0, a.M);
            a.attn_out = attn_ptr(0);
            a.attn_stride = astride;
            VDM_TRY(launch_decode(a, dec->dtype, st));
            if (sb) { sb->resolution[0] = R; sb->decoded[0] = a.M; }
        }
        for (int l = 0; l + 1 < L; ++l) {
            const int R = pl.R[l], R2 = 2 * R;
            const int nb = R / 4;
            const int nw = nb * nb * nb;
            uint64_t* words = at<uint64_t>(ws, pl.off_words);
            int32_t* word_off = at<int32_t>(ws, pl.off_word_off);
            int32_t* tile_ids = at<int32_t>(ws, pl.off_tile_ids);
            int32_t* tile_off = at<int32_t>(ws, pl.off_tile_off);
            int32_t* counts = at<int32_t>(ws, pl.off_counts) + 4 * (l + 1);
            int32_t* scan_tmp = at<int32_t>(ws, pl.off_scan);
            int32_t* plist = at<int32_t>(ws, pl.off_plist);
            int32_t* qorder = at<int32_t>(ws, pl.off_qorder);
            int32_t* sel = at<int32_t>(ws, pl.off_sel);
            // near-surface rule: |tSDF| < threshold with a tSDF head, else |f| < float32(4 / R)
            VDM_TRY(launch_mark_dilate(grid[l], tsdf ? tgrid[l] : grid[l], R,
                                       tsdf ? p->tsdf_threshold : (float)(4.0 / (double)R), words,
                                       at<uint64_t>(ws, pl.off_bits), st));
            VDM_TRY(launch_compact(words, nw, R, word_off, tile_ids, tile_off, plist, counts, scan_tmp, st));
            // the inherit fill needs no count: it runs while the counts travel to the host
            VDM_TRY(launch_fill(grid[l], R, grid[l + 1], st));
            if (tgrid[l + 1]) VDM_TRY(launch_fill(tgrid[l], R, tgrid[l + 1], st));
            int32_t hc[2] = {0, 0};
            VDM_CUDA_TRY(cudaMemcpyAsync(hc, counts, sizeof(hc), cudaMemcpyDeviceToHost, st));
            VDM_CUDA_TRY(cudaStreamSynchronize(st));
            VDM_TRY(tc_check_error());
            const int Mp = hc[0], T = hc[1];
            if (dbg && dbg->active[l])
                VDM_CUDA_TRY(cudaMemcpyAsync(dbg->active[l] + (size_t)b * nw, words, (size_t)nw * 8,
                                             cudaMemcpyDeviceToDevice, st));
            const int64_t vox2 = (int64_t)R2 * R2 * R2;
            float* decg = dbg_ptr(dbg ? dbg->dec : nullptr, l + 1, vox2);
            if (sb) {
                sb->resolution[l + 1] = R2;
                sb->active_parents[l + 1] = Mp;
                sb->tiles[l + 1] = T;
            }
            if (Mp == 0) continue;
            if (!p->adaptive) {
                DecodeArgs a = base;
                a.work = kWorkFlat;
                a.qmode = kQueryChildren;
                a.R = R2;
                a.plist = plist;
                a.M = 8 * (int64_t)Mp;
                a.grid = grid[l + 1];
                a.tsdf_grid = tgrid[l + 1];
                a.dec_grid = decg;
                a.attn_out = attn_ptr(l + 1);
                a.attn_stride = astride;
                VDM_TRY(launch_decode(a, dec->dtype, st));
                if (sb) sb->decoded[l + 1] = a.M;
                continue;
            }
            const uint64_t salt = splitmix64(p->seed ^ ((uint64_t)(l + 1) << 32));
            int32_t* sel_tiles = at<int32_t>(ws, pl.off_seltiles);
            float* probe_ml = at<float>(ws, pl.off_ml);
            const bool sel_tc = select_tc_supported(dec->C, p->n_probe, N, dec->dtype);
            VDM_CUDA_TRY(cudaMemsetAsync(counts + 2, 0, 2 * sizeof(int32_t), st));
            int32_t* dense_q = at<int32_t>(ws, pl.off_dense);
            int32_t* dense_ml = at<int32_t>(ws, pl.off_dense_ml);
            VDM_TRY(launch_probe_order(tile_off, T, plist, R2, p->n_probe, salt, qorder, counts + 2, sel_tiles,
                                       dense_q, dense_ml, st));
            const int dbg_rows = dbg ? (int)std::min<int64_t>(T, dbg->max_tiles) : 0;
            if (dbg && dbg->probes[l + 1] && dbg_rows > 0)
                VDM_TRY(launch_probe_export(tile_off, dbg_rows, plist, qorder, R2, p->n_probe,
                                            dbg->probes[l + 1] + (size_t)b * dbg->max_tiles * p->n_probe,
                                            st));
            float* score_dbg = (dbg && dbg->scores[l + 1] && dbg_rows > 0)
                                   ? dbg->scores[l + 1] + (size_t)b * dbg->max_tiles * N
                                   : nullptr;
            DecodeArgs a = base;
            a.qmode = kQueryChildren;
            a.R = R2;
            a.plist = plist;
            a.qorder = qorder;
            a.tile_off = tile_off;
            a.T = T;
            a.n_probe = p->n_probe;
            a.grid = grid[l + 1];
            a.tsdf_grid = tgrid[l + 1];
            a.dec_grid = decg;
            a.attn_out = attn_ptr(l + 1);
            a.attn_stride = astride;
            // dense pass: probes and small sub-volumes, packed into one flat list
            // (exports the probes' softmax statistics for the scoring kernel)
            {
                DecodeArgs d = a;
                d.work = kWorkFlat;
                d.qlist = dense_q;
                d.M = std::min<int64_t>(8 * (int64_t)Mp, (int64_t)T * std::min(p->n_probe, 512));
                d.M_dev = counts + 3;
                d.probe_ml = sel_tc ? probe_ml : nullptr;
                d.ml_slot = sel_tc ? dense_ml : nullptr;
                VDM_TRY(launch_decode(d, dec->dtype, st));
            }
            // selection
            if (sel_tc) {
                SelectTcLaunch L{};
                L.C = dec->C; L.H = dec->H; L.N = N;
                L.Wq = dec->Wq; L.bq = dec->bq; L.K = K;
                L.T = T;
                L.n_sel = counts + 2;
                L.sel_tiles = sel_tiles;
                L.tile_off = tile_off; L.plist = plist; L.qorder = qorder;
                L.probe_ml = probe_ml;
                L.R = R2; L.n_probe = p->n_probe; L.top_k = pl.k;
                L.sel = sel;
                L.score_out = score_dbg;
                L.score_rows = dbg_rows;
                VDM_TRY(launch_select_tc(L, st));
            } else {
            SelectArgs s;
            memset(&s, 0, sizeof(s));
            s.C = dec->C; s.H = dec->H; s.N = N;
            s.Wq = dec->Wq; s.bq = dec->bq; s.K = K;
            s.T = T;
            s.tile_off = tile_off; s.plist = plist; s.qorder = qorder; s.R = R2;
            s.n_probe = p->n_probe;
            s.top_k = pl.k;
            s.sel = sel;
            // the CUDA-core selection writes a score row for every sub-volume it scores
            s.score = (score_dbg && T <= dbg_rows) ? score_dbg : nullptr;
            VDM_TRY(launch_select(s, dec->dtype, st));
            }
            // sparse pass: the remaining queries over the selected tokens
            if (p->n_probe < 512) {
                a.work = kWorkTileSparse;
                a.sel = sel;
                a.ksel = pl.k;
                int32_t* units = at<int32_t>(ws, pl.off_units);
                int32_t* units_n = at<int32_t>(ws, pl.off_units_n);
                VDM_TRY(launch_sparse_units(tile_off, T, p->n_probe, kTcTile, units, units_n, st));
                a.unit_list = units;
                a.n_units_dev = units_n;
                VDM_TRY(launch_decode(a, dec->dtype, st));
            }
            if (dbg && dbg->tile_ids[l + 1] && dbg->max_tiles > 0) {
                const int64_t nt = T < dbg->max_tiles ? T : dbg->max_tiles;
                VDM_CUDA_TRY(cudaMemcpyAsync(dbg->tile_ids[l + 1] + (size_t)b * dbg->max_tiles, tile_ids,
                                             nt * 4, cudaMemcpyDeviceToDevice, st));
                if (dbg->sel[l + 1])
                    VDM_CUDA_TRY(cudaMemcpyAsync(dbg->sel[l + 1] + (size_t)b * dbg->max_tiles * pl.k, sel,
                                                 nt * pl.k * 4, cudaMemcpyDeviceToDevice, st));
            }
            if (sb) sb->decoded[l + 1] = 8 * (int64_t)Mp;
        }
        if (sb && p->adaptive && L > 1) {
            int32_t hc[4 * VDM_MAX_LEVELS];
            VDM_CUDA_TRY(cudaMemcpyAsync(hc, at<int32_t>(ws, pl.off_counts), sizeof(int32_t) * 4 * L,
                                         cudaMemcpyDeviceToHost, st));
            VDM_CUDA_TRY(cudaStreamSynchronize(st));
            for (int l = 1; l < L; ++l) {
                if (sb->active_parents[l] == 0) continue;
                sb->selected_tiles[l] = hc[4 * l + 2];
                sb->probes[l] = hc[4 * l + 3];
            }
        }
        if (dbg) {
            for (int l = 0; l < L; ++l) {
                const size_t v = (size_t)pl.R[l] * pl.R[l] * pl.R[l];
                if (dbg->grid[l])
                    VDM_CUDA_TRY(cudaMemcpyAsync(dbg->grid[l] + (size_t)b * v, grid[l], v * 4,
                                                 cudaMemcpyDeviceToDevice, st));
                if (tsdf && l < L - 1 && dbg->tsdf[l])
                    VDM_CUDA_TRY(cudaMemcpyAsync(dbg->tsdf[l] + (size_t)b * v, tgrid[l], v * 4,
                                                 cudaMemcpyDeviceToDevice, st));
            }
        }
    }
    // the last level's kernels: their bounded-wait status reaches this caller too
    VDM_CUDA_TRY(cudaStreamSynchronize(st));
    return tc_check_error();
}

}  // extern "C"
