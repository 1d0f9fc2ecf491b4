// K/V projection and the fused SIMT (CUDA-core, fp32 arithmetic) decoder.
//
// The decoder is the vecset decoder of FlashVDM ("Unleashing Vecset Diffusion
// Model for Fast Shape Generation", aipaper.cc summary, section 3: cross-
// attention from query points to the latent set, then the SDF): Fourier
// embedding -> Q projection -> multi-head cross-attention (online softmax over
// token blocks) -> output projection + residual -> LN + GELU MLP + residual ->
// LN + SDF head (+ optional analytic sphere term).  One CTA decodes QT query
// points with every intermediate in shared memory; nothing but the final
// value goes back to global memory.
//
// This kernel is the product path for float32 decoders; bf16 decoders read
// bf16 weights and K/V and compute in float32 here.
#include "vdm_internal.cuh"

namespace vdm {
namespace {

constexpr int QT = 32;        // queries per CTA
constexpr int NT = 256;       // threads per CTA
constexpr int KB = 64;        // tokens per K/V block
constexpr int KLD = 65;       // padded row stride of staged K/V (bank spread)
constexpr int HC = 128;       // MLP hidden chunk

// acc[c][r] += sum_k xs[r][k] * W[col_c][k]   (NC columns, QT rows; xs in smem)
template <int NC, int NR, typename T>
__device__ __forceinline__ void rows_x_cols(const float* xs, int ldx, const T* w, int ldw,
                                            const int* cols, int K, float (&acc)[NC][NR]) {
    for (int k = 0; k < K; k += 4) {
        float4 wv[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) wv[c] = load4(w + (size_t)cols[c] * ldw + k);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            float4 x = *reinterpret_cast<const float4*>(xs + r * ldx + k);
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                float a = acc[c][r];
                a = fmaf(x.x, wv[c].x, a);
                a = fmaf(x.y, wv[c].y, a);
                a = fmaf(x.z, wv[c].z, a);
                a = fmaf(x.w, wv[c].w, a);
                acc[c][r] = a;
            }
        }
    }
}

// Row-wise LayerNorm of rows [0, nrows) of src (width C) into dst (may alias).
__device__ void layer_norm_rows(const float* src, float* dst, int ld, int nrows, int C,
                                const float* g, const float* b, bool affine_only_copy) {
    int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < nrows; r += NT / 32) {
        const float* x = src + r * ld;
        float* y = dst + r * ld;
        if (affine_only_copy) {
            for (int c = lane; c < C; c += 32) y[c] = x[c];
            continue;
        }
        float s = 0.f;
        for (int c = lane; c < C; c += 32) s += x[c];
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        float mu = s / (float)C;
        float v = 0.f;
        for (int c = lane; c < C; c += 32) {
            float d = x[c] - mu;
            v = fmaf(d, d, v);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        float rs = rsqrtf(v / (float)C + kLnEps);
        for (int c = lane; c < C; c += 32) y[c] = (x[c] - mu) * rs * g[c] + b[c];
    }
}

// ------------------------------------------------------------------ K/V projection
constexpr int KV_ROWS = 16;

template <typename T>
__global__ void __launch_bounds__(NT) kv_kernel(KvArgs a) {
    extern __shared__ float smem[];
    const int C = a.C, N = a.N;
    const int ld = C + 4;
    float* zs = smem;  // [KV_ROWS][ld]
    const int n0 = blockIdx.x * KV_ROWS;
    const int nrows = min(KV_ROWS, N - n0);
    for (int i = threadIdx.x; i < KV_ROWS * C; i += NT) {
        int r = i / C, c = i - r * C;
        zs[r * ld + c] = r < nrows ? a.z[(size_t)(n0 + r) * C + c] : 0.f;
    }
    __syncthreads();
    layer_norm_rows(zs, zs, ld, nrows, C, a.g, a.b, false);
    __syncthreads();
    const T* Wk = static_cast<const T*>(a.Wk);
    const T* Wv = static_cast<const T*>(a.Wv);
    T* K = static_cast<T*>(a.K);
    T* V = static_cast<T*>(a.V);
    for (int col = threadIdx.x; col < 2 * C; col += NT) {
        const bool isv = col >= C;
        const int c = isv ? col - C : col;
        int cols[1] = {c};
        float acc[1][KV_ROWS] = {};
        rows_x_cols<1, KV_ROWS>(zs, ld, isv ? Wv : Wk, C, cols, C, acc);
        const float bias = isv ? a.bv[c] : a.bk[c];
        const int h = c >> 6, d = c & 63;
        T* dst = isv ? V : K;
        for (int r = 0; r < nrows; ++r)
            dst[((size_t)h * N + n0 + r) * kHeadDim + d] = from_f<T>(acc[0][r] + bias);
    }
}

// ------------------------------------------------------------------ decoder
struct Smem {
    float* xq;    // [QT][ldc]  residual stream (q, x1, x2)
    float* buf;   // [QT][ldc]  attention output, then LN(x1)
    float* hid;   // [QT][HC+4] MLP hidden chunk
    float* pe;    // [QT][68]   embedding
    float* kb;    // [KB][KLD]  staged keys
    float* vb;    // [KB][KLD]  staged values
    float* pb;    // [QT][KB+1] softmax weights of the block
    float* ml;    // [QT][2]    running max / sum
    float* pts;   // [QT][4]    query points
    int64_t* vox; // [QT]       voxel index (or -1)
    int* qid;     // [QT]       output slot (flat) or -1
    int* tok;     // [KB]       gathered token ids
};

__host__ __device__ inline size_t decode_smem_bytes(int C) {
    int ldc = C + 4;
    size_t f = (size_t)QT * ldc * 2 + QT * (HC + 4) + QT * 68 + 2 * KB * KLD + QT * (KB + 1) +
               QT * 2 + QT * 4;
    return f * 4 + QT * 8 + QT * 4 + KB * 4 + 64;
}

template <typename T>
__global__ void __launch_bounds__(NT) decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) float smem[];
    const int C = a.C, H = a.H, F = a.F, N = a.N;
    const int ldc = C + 4;
    const int tid = threadIdx.x;
    Smem s;
    s.xq = smem;
    s.buf = s.xq + QT * ldc;
    s.hid = s.buf + QT * ldc;
    s.pe = s.hid + QT * (HC + 4);
    s.kb = s.pe + QT * 68;
    s.vb = s.kb + KB * KLD;
    s.pb = s.vb + KB * KLD;
    s.ml = s.pb + QT * (KB + 1);
    s.pts = s.ml + QT * 2;
    s.vox = reinterpret_cast<int64_t*>(s.pts + QT * 4);
    s.qid = reinterpret_cast<int*>(s.vox + QT);
    s.tok = s.qid + QT;

    // ---------------- which queries does this CTA own?
    int nq = 0;
    const int32_t* sel = nullptr;
    int64_t qbeg = 0;   // first query slot (flat) or qorder position (tiles)
    if (a.work == kWorkFlat) {
        const int64_t M = a.M_dev ? (int64_t)*a.M_dev : a.M;
        qbeg = (int64_t)blockIdx.x * QT;
        if (qbeg >= M) return;
        nq = (int)(M - qbeg < QT ? M - qbeg : QT);
    } else {
        const int t = blockIdx.x / a.slots, sl = blockIdx.x - t * a.slots;
        if (t >= a.T) return;
        const int cnt = 8 * (a.tile_off[t + 1] - a.tile_off[t]);
        const int base = 8 * a.tile_off[t];
        int lo, n;
        if (a.work == kWorkTileDense) {
            lo = 0;
            n = min(cnt, a.n_probe);
        } else {
            lo = a.n_probe;
            n = cnt > a.n_probe ? cnt - a.n_probe : 0;
            sel = a.sel + (size_t)t * a.ksel;
        }
        const int first = lo + sl * QT;
        if (first >= lo + n) return;
        nq = min(QT, lo + n - first);
        qbeg = base + first;
    }
    if (tid < QT) {
        float p[3] = {0.f, 0.f, 0.f};
        int64_t v = -1;
        int q = -1;
        if (tid < nq) {
            const int64_t slot = qbeg + tid;
            if (a.qmode == kQueryXyz) {
                p[0] = a.xyz[slot * 3];
                p[1] = a.xyz[slot * 3 + 1];
                p[2] = a.xyz[slot * 3 + 2];
                q = (int)slot;
            } else if (a.qmode == kQueryGrid) {
                v = slot;
                voxel_point(v, a.R, p);
                q = (int)slot;
            } else {
                const int64_t pos = a.qlist ? (int64_t)a.qlist[slot] : slot;
                const int e = a.qorder ? a.qorder[pos] : (int)pos;
                v = child_index(a.plist[e >> 3], e & 7, a.R);
                voxel_point(v, a.R, p);
                q = (int)slot;
            }
        }
        s.pts[tid * 4] = p[0];
        s.pts[tid * 4 + 1] = p[1];
        s.pts[tid * 4 + 2] = p[2];
        s.vox[tid] = v;
        s.qid[tid] = q;
    }
    __syncthreads();
    // ---------------- embedding
    for (int i = tid; i < QT * 64; i += NT) {
        const int r = i >> 6, l = i & 63;
        float p[3] = {s.pts[r * 4], s.pts[r * 4 + 1], s.pts[r * 4 + 2]};
        s.pe[r * 68 + l] = pe_lane(p, l);
    }
    __syncthreads();
    const T* Wq = static_cast<const T*>(a.Wq);
    const T* Wo = static_cast<const T*>(a.Wo);
    const T* W1 = static_cast<const T*>(a.W1);
    const T* W2 = static_cast<const T*>(a.W2);
    const T* Kg = static_cast<const T*>(a.K);
    const T* Vg = static_cast<const T*>(a.V);

    // ---------------- q = Wq pe + bq  -> xq
    for (int c0 = tid; c0 < C; c0 += NT) {
        int cols[1] = {c0};
        float acc[1][QT] = {};
        rows_x_cols<1, QT>(s.pe, 68, Wq, kPeLanes, cols, kPeLanes, acc);
        const float bb = a.bq[c0];
#pragma unroll
        for (int r = 0; r < QT; ++r) s.xq[r * ldc + c0] = acc[0][r] + bb;
    }
    __syncthreads();

    // ---------------- multi-head cross-attention -> buf
    const int nk = sel ? a.ksel : N;
    const float scale = 0.125f;
    // thread roles: score/softmax: query r = tid/8, token lane jj = tid%8 (8 tokens each)
    //               PV: query r = tid/8, dims (tid%8)*8 .. +8
    const int r8 = tid >> 3, j8 = tid & 7;
    for (int h = 0; h < H; ++h) {
        float o[8] = {};
        float m_run = -INFINITY, l_run = 0.f;
        const float* qh = s.xq + r8 * ldc + h * kHeadDim;
        for (int j0 = 0; j0 < nk; j0 += KB) {
            const int nb = min(KB, nk - j0);
            __syncthreads();   // previous block fully consumed
            if (tid < KB) s.tok[tid] = tid < nb ? (sel ? sel[j0 + tid] : j0 + tid) : 0;
            __syncthreads();
            for (int i = tid; i < KB * 16; i += NT) {
                const int jr = i >> 4, d4 = (i & 15) * 4;
                float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
                if (jr < nb) {
                    const size_t row = ((size_t)h * N + s.tok[jr]) * kHeadDim + d4;
                    kv = load4(Kg + row);
                    vv = load4(Vg + row);
                }
                float* kd = s.kb + jr * KLD + d4;
                float* vd = s.vb + jr * KLD + d4;
                kd[0] = kv.x; kd[1] = kv.y; kd[2] = kv.z; kd[3] = kv.w;
                vd[0] = vv.x; vd[1] = vv.y; vd[2] = vv.z; vd[3] = vv.w;
            }
            __syncthreads();
            // scores for tokens jj + 8 i
            float sc[8];
            float bmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int j = j8 + 8 * i;
                const float* kr = s.kb + j * KLD;
                float acc = 0.f;
#pragma unroll 16
                for (int d = 0; d < kHeadDim; ++d) acc = fmaf(qh[d], kr[d], acc);
                sc[i] = j < nb ? acc * scale : -INFINITY;
                bmax = fmaxf(bmax, sc[i]);
            }
#pragma unroll
            for (int off = 4; off; off >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, off));
            const float m_new = fmaxf(m_run, bmax);
            const float corr = expf(m_run - m_new);   // exp(-inf) = 0 on the first block
            float psum = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float p = expf(sc[i] - m_new);
                psum += p;
                s.pb[r8 * (KB + 1) + j8 + 8 * i] = p;
            }
#pragma unroll
            for (int off = 4; off; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
            l_run = l_run * corr + psum;
            m_run = m_new;
#pragma unroll
            for (int d = 0; d < 8; ++d) o[d] *= corr;
            __syncwarp();
            // o[d] += sum_j p[r][j] v[j][d] ; p row r written by the 8 lanes of this group
            const float* prow = s.pb + r8 * (KB + 1);
            for (int j = 0; j < nb; ++j) {
                const float p = prow[j];
                const float* vr = s.vb + j * KLD + j8 * 8;
#pragma unroll
                for (int d = 0; d < 8; ++d) o[d] = fmaf(p, vr[d], o[d]);
            }
        }
        __syncthreads();
        const float inv = 1.0f / l_run;
#pragma unroll
        for (int d = 0; d < 8; ++d) s.buf[r8 * ldc + h * kHeadDim + j8 * 8 + d] = o[d] * inv;
    }
    __syncthreads();
    if (a.attn_out) {   // debug export of the attention output at sampled voxels
        for (int i = tid; i < QT * C; i += NT) {
            const int r = i / C, c = i - r * C;
            const int64_t v = s.vox[r];
            if (r < nq && v >= 0 && v % a.attn_stride == 0)
                a.attn_out[(size_t)(v / a.attn_stride) * C + c] = s.buf[r * ldc + c];
        }
    }

    // ---------------- x1 = q + Wo a + bo
    for (int c0 = tid; c0 < C; c0 += NT) {
        int cols[1] = {c0};
        float acc[1][QT] = {};
        rows_x_cols<1, QT>(s.buf, ldc, Wo, C, cols, C, acc);
        const float bb = a.bo[c0];
#pragma unroll
        for (int r = 0; r < QT; ++r) s.xq[r * ldc + c0] += acc[0][r] + bb;
    }
    __syncthreads();
    // ---------------- LN1 -> buf
    layer_norm_rows(s.xq, s.buf, ldc, QT, C, a.ln1_g, a.ln1_b, !a.query_ln);
    __syncthreads();
    // ---------------- MLP in hidden chunks: xq += W2 GELU(W1 buf + b1)
    for (int f0 = 0; f0 < F; f0 += HC) {
        const int hc = min(HC, F - f0);   // F is a multiple of 64
        // hidden: thread -> hidden unit tid%HC, rows half (tid/HC)*16 .. +16
        {
            const int fh = tid % HC, rh = (tid / HC) * (QT / 2);
            if (fh < hc) {
                int cols[1] = {f0 + fh};
                float acc[1][QT / 2] = {};
                rows_x_cols<1, QT / 2>(s.buf + rh * ldc, ldc, W1, C, cols, C, acc);
                const float bb = a.b1[f0 + fh];
#pragma unroll
                for (int r = 0; r < QT / 2; ++r) s.hid[(rh + r) * (HC + 4) + fh] = gelu_erf(acc[0][r] + bb);
            }
        }
        __syncthreads();
        for (int c0 = tid; c0 < C; c0 += NT) {
            int cols[1] = {c0};
            float acc[1][QT] = {};
            rows_x_cols<1, QT>(s.hid, HC + 4, W2 + f0, F, cols, hc, acc);
#pragma unroll
            for (int r = 0; r < QT; ++r) s.xq[r * ldc + c0] += acc[0][r];
        }
        __syncthreads();
    }
    for (int i = tid; i < QT * C; i += NT) {
        const int r = i / C, c = i - r * C;
        s.xq[r * ldc + c] += a.b2[c];
    }
    __syncthreads();
    if (a.feat_out) {   // the block output itself (vecset encoding)
        for (int i = tid; i < nq * C; i += NT) {
            const int r = i / C, c = i - r * C;
            a.feat_out[(size_t)s.qid[r] * C + c] = s.xq[r * ldc + c];
        }
    }
    // ---------------- LN2 + head
    layer_norm_rows(s.xq, s.buf, ldc, QT, C, a.ln2_g, a.ln2_b, !a.query_ln);
    __syncthreads();
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp; r < nq; r += NT / 32) {
            float acc = 0.f, acc_t = 0.f;
            for (int c = lane; c < C; c += 32) {
                acc = fmaf(s.buf[r * ldc + c], a.w_head[c], acc);
                if (a.w_tsdf) acc_t = fmaf(s.buf[r * ldc + c], a.w_tsdf[c], acc_t);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                acc += __shfl_xor_sync(0xffffffffu, acc, o);
                acc_t += __shfl_xor_sync(0xffffffffu, acc_t, o);
            }
            if (lane == 0) {
                const float dec = acc + a.b_head[0];
                float val = dec, sph = 0.f;
                if (a.spheres) {
                    float p[3] = {s.pts[r * 4], s.pts[r * 4 + 1], s.pts[r * 4 + 2]};
                    sph = sphere_union(p, a.spheres, a.n_spheres);
                    val = sph + a.dec_scale * tanhf(dec);
                }
                if (a.out) a.out[s.qid[r]] = val;
                const int64_t v = s.vox[r];
                if (v >= 0) {
                    if (a.grid) a.grid[v] = val;
                    if (a.dec_grid) a.dec_grid[v] = dec;
                    if (a.tsdf_grid) a.tsdf_grid[v] = tsdf_value(acc_t + a.b_tsdf[0], sph, a);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ point features (encoder)
// u[m][c] = sum_l W_in[c][l] pe_l(p_m) + b_in[c]: 16 points per CTA, embedding in shared memory
template <typename T>
__global__ void __launch_bounds__(NT) point_feature_kernel(const float* __restrict__ pts, int M, int C,
                                                           const T* __restrict__ W, const float* __restrict__ b,
                                                           float* __restrict__ u) {
    __shared__ __align__(16) float pe[KV_ROWS * 68];
    const int m0 = blockIdx.x * KV_ROWS;
    const int n = min(KV_ROWS, M - m0);
    for (int i = threadIdx.x; i < KV_ROWS * 64; i += NT) {
        const int r = i >> 6, l = i & 63;
        float p[3] = {0.f, 0.f, 0.f};
        if (r < n) {
            p[0] = pts[(size_t)(m0 + r) * 3];
            p[1] = pts[(size_t)(m0 + r) * 3 + 1];
            p[2] = pts[(size_t)(m0 + r) * 3 + 2];
        }
        pe[r * 68 + l] = pe_lane(p, l);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += NT) {
        int cols[1] = {c};
        float acc[1][KV_ROWS] = {};
        rows_x_cols<1, KV_ROWS>(pe, 68, W, kPeLanes, cols, kPeLanes, acc);
        for (int r = 0; r < n; ++r) u[(size_t)(m0 + r) * C + c] = acc[0][r] + b[c];
    }
}

}  // namespace

vdm_status launch_point_features(const float* points, int M, int C, const void* W_in, const float* b_in, float* u,
                                 vdm_dtype dt, cudaStream_t st) {
    const dim3 grid((M + KV_ROWS - 1) / KV_ROWS);
    if (dt == VDM_F32)
        point_feature_kernel<float><<<grid, NT, 0, st>>>(points, M, C, static_cast<const float*>(W_in), b_in, u);
    else
        point_feature_kernel<__nv_bfloat16><<<grid, NT, 0, st>>>(points, M, C,
                                                                 static_cast<const __nv_bfloat16*>(W_in), b_in, u);
    return check_launch("point_feature_kernel");
}

vdm_status launch_precompute_kv(const KvArgs& a, vdm_dtype dt, cudaStream_t st) {
    const size_t sm = (size_t)KV_ROWS * (a.C + 4) * 4;
    dim3 grid((a.N + KV_ROWS - 1) / KV_ROWS);
    prof_begin(kProfKv, st);
    if (dt == VDM_F32) {
        kv_kernel<float><<<grid, NT, sm, st>>>(a);
    } else {
        kv_kernel<__nv_bfloat16><<<grid, NT, sm, st>>>(a);
    }
    prof_end(kProfKv, st);
    return check_launch("kv_kernel");
}

vdm_status launch_decode_simt(const DecodeArgs& a, vdm_dtype dt, int /*hint*/, cudaStream_t st) {
    int64_t ctas;
    if (a.work == kWorkFlat) {
        if (a.M <= 0) return VDM_OK;
        ctas = (a.M + QT - 1) / QT;
    } else {
        if (a.T <= 0) return VDM_OK;
        ctas = (int64_t)a.T * a.slots;
    }
    if (ctas > 0x7fffffff) return fail(VDM_ERR_UNSUPPORTED, "too many queries for one launch");
    const size_t sm = decode_smem_bytes(a.C);
    cudaError_t e = dt == VDM_F32
        ? cudaFuncSetAttribute(decode_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)
        : cudaFuncSetAttribute(decode_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "decode_kernel smem attribute: %s", cudaGetErrorString(e));
    prof_begin(kProfDecode, st);
    if (dt == VDM_F32) {
        decode_kernel<float><<<(unsigned)ctas, NT, sm, st>>>(a);
    } else {
        decode_kernel<__nv_bfloat16><<<(unsigned)ctas, NT, sm, st>>>(a);
    }
    prof_end(kProfDecode, st);
    return check_launch("decode_kernel");
}

int decode_simt_chunk() { return QT; }

}  // namespace vdm
