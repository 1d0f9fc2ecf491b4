// Adaptive KV selection on the tensor cores: probe scoring and Top-K.
//
// FlashVDM ("Unleashing Vecset Diffusion Model for Fast Shape Generation",
// aipaper.cc summary, section 4.1 item 2, steps 2-4): sampled queries of each
// sub-volume score all vecset tokens by attention; the Top-K tokens are kept.
//
// score_t[j] = sum over the probes p of sub-volume t and heads h of
//              softmax_h(q_p K_h^T / 8)_j
//
// The probes were already decoded with full attention by the dense pass of the
// level, which exported each probe's per-head softmax maximum m and sum l (in
// log2 units, against the same bf16 Q and K).  One pass suffices here:
// S = Q K^T on the tensor cores (TMEM), P = 2^(S - m) / l in registers, summed
// over the heads in registers (key blocks outer, heads inner: the packed Q of
// every head stays in TMEM), then per key block the column sums over each
// sub-volume's probe rows by a warp transpose-reduce (5 shuffle rounds; lane L
// ends with column L of the warp's 32) plus a fixed-order sum over the sub-volume's warps
// -- deterministic.  Then a radix select of the k largest scores (ties to the
// smaller token) per sub-volume, in shared memory.
//
// Rows: 128 TMEM lanes hold 128 / n_probe sub-volumes' probes (n_probe in
// {32, 64, 128}).  Roles: warps 0-15 compute in four warpgroups (thread (g, r)
// owns row r and the 32 columns [32g, 32g+32) of each 128-token block, so every
// SM sub-partition runs four compute warps to hide the TMEM and exponential
// latencies), warp 16 MMA issue, warp 17 TMA.
#include <cuda.h>

#include "tc_ptx.cuh"
#include "vdm_internal.cuh"

namespace vdm {

vdm_status make_bf16_map(CUtensorMap* m, const void* base, int64_t rows, int cols, int box_rows, int box_cols);
int* tc_error_word();

namespace {

using namespace ptx;

constexpr int NT = 576;
constexpr int NCOMP = 512;   // compute threads: four warpgroups, 32 of the 128 columns of a block each
constexpr int WARP_MMA = 16, WARP_PROD = 17;
constexpr int SLOT = 16384;
constexpr int NS = 6;
constexpr float kLog2e = 1.4426950408889634f;
// TMEM: packed bf16 Q of head h in [32h, 32h+32) (up to 8 heads); the S double buffer in
// [256, 384) and [384, 512), which first holds the fp32 Q projections of up to 4 heads
// (64 columns each) while they are packed
constexpr uint32_t T_QP = 0, T_S0 = 256, T_QA = 256;
constexpr int QROUND = 4;   // heads projected per round

struct SelArgs {
    int C, H, N;
    const void* bq_unused;
    const float* bq;
    int n_sel_max;                 // capacity of the tile list
    const int32_t* n_sel;          // device: number of tiles to score
    const int32_t* sel_tiles;      // device: their ids
    const int32_t* tile_off;       // [T+1] parent offsets
    const int32_t* plist;
    const int32_t* qorder;
    const float* probe_xyz;        // probes given as points (or NULL: hierarchical children)
    const int32_t* probe_off;      // [T+1] with probe_xyz: probes of tile t are [probe_off[t], probe_off[t+1])
    const float* probe_ml;         // [T][n_probe][H][2]
    int R;
    int n_probe;
    int tpu;                       // sub-volumes per unit = 128 / n_probe
    int top_k;
    int32_t* sel;                  // [T][top_k]
    float* score_out;              // debug: [score_rows][N] scores by tile id, or NULL
    int score_rows;
    int* err;
    long long timeout;
};

struct Shared {
    uint64_t full[NS], empty[NS];
    uint64_t bar_q, bar_s[2];                  // MMA commits
    uint64_t bar_pe, bar_qc, bar_p[2], bar_cs; // compute arrivals (128)
    uint32_t tmem_base;
    int abort;
    int hist[256];
    int red[4];
    int wsum[NCOMP / 32];
};

struct Waiter {
    Shared* sh;
    int* err;
    long long timeout;
    __device__ bool wait(uint64_t* bar, uint32_t& phase, int site) {
        const uint32_t b = smem_u32(bar);
        long long t0 = 0;
        for (uint32_t it = 0;; ++it) {
            if (mbar_try_wait(b, phase)) {
                phase ^= 1;
                return true;
            }
            if ((it & 63) == 63) {
                if (*reinterpret_cast<volatile int*>(&sh->abort)) return false;
                const long long t = clock64();
                if (t0 == 0) t0 = t;
                else if (t - t0 > timeout) {
                    *reinterpret_cast<volatile int*>(&sh->abort) = 1;
                    atomicCAS(err, 0, site);
                    return false;
                }
            }
        }
    }
};

__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int c) {
    return base + r * 128 + ((c ^ (r & 7)) << 4);
}

// Sum of v over the 32 lanes for each of 32 columns; lane L returns the sum of column L.
__device__ __forceinline__ float warp_colsum32(const float (&v)[32], int lane) {
    float a16[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool up = lane & 16;
        const float send = up ? v[i] : v[i + 16];
        const float keep = up ? v[i + 16] : v[i];
        a16[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float a8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 8;
        const float send = up ? a16[i] : a16[i + 8];
        const float keep = up ? a16[i + 8] : a16[i];
        a8[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float a4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 4;
        const float send = up ? a8[i] : a8[i + 4];
        const float keep = up ? a8[i + 4] : a8[i];
        a4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    float a2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 2;
        const float send = up ? a4[i] : a4[i + 2];
        const float keep = up ? a4[i + 2] : a4[i];
        a2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    const bool up = lane & 1;
    return (up ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, up ? a2[0] : a2[1], 1);
}

__global__ void __launch_bounds__(NT, 1)
select_tc_kernel(const __grid_constant__ CUtensorMap tm_wq64, const __grid_constant__ CUtensorMap tm_k,
                 const SelArgs a) {
    extern __shared__ uint8_t dyn_raw[];
    __shared__ Shared sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, N = a.N, np = a.n_probe, tpu = a.tpu;
    const int nb = (N + 127) / 128;
    const uint32_t dyn0 = (smem_u32(dyn_raw) + 1023u) & ~1023u;
    const uint32_t s_pe = dyn0;
    const uint32_t s_ring = s_pe + 16384;
    float* score = reinterpret_cast<float*>(dyn_raw + (dyn0 - smem_u32(dyn_raw)) + 16384 + NS * SLOT);  // [tpu][N]
    float* part = score + (size_t)tpu * N;    // [2][16 warps][32]
    Waiter W{&sh, a.err, a.timeout};

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(smem_u32(&sh.full[i]), 1);
            mbar_init(smem_u32(&sh.empty[i]), 1);
        }
        mbar_init(smem_u32(&sh.bar_q), 1);
        mbar_init(smem_u32(&sh.bar_s[0]), 1);
        mbar_init(smem_u32(&sh.bar_s[1]), 1);
        mbar_init(smem_u32(&sh.bar_pe), NCOMP);
        mbar_init(smem_u32(&sh.bar_qc), NCOMP);
        mbar_init(smem_u32(&sh.bar_p[0]), NCOMP);
        mbar_init(smem_u32(&sh.bar_p[1]), NCOMP);
        mbar_init(smem_u32(&sh.bar_cs), NCOMP);
        sh.abort = 0;
        fence_mbar_init();
        fence_proxy_async();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sh.tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int n_sel = *a.n_sel < a.n_sel_max ? *a.n_sel : a.n_sel_max;
    const int n_units = (n_sel + tpu - 1) / tpu;

    if (warp == WARP_PROD) {
        // ------------------------------------------------------------ producer
        uint32_t ring_head = 0;
        bool ok = true;
        auto push = [&](const CUtensorMap* m, int y, uint32_t bytes) -> bool {
            const int slot = ring_head % NS;
            if (ring_head >= (uint32_t)NS) {
                uint32_t ph = ((ring_head / NS) + 1) & 1;
                if (!W.wait(&sh.empty[slot], ph, 80)) return false;
            }
            ++ring_head;
            if (lane == 0) {
                const uint32_t fb = smem_u32(&sh.full[slot]);
                mbar_expect_tx(fb, bytes);
                tma_load_2d(s_ring + slot * SLOT, m, 0, y, fb);
            }
            __syncwarp();
            return true;
        };
        for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
            for (int h = 0; h < H && ok; ++h) ok = push(&tm_wq64, h * 64, 64 * 128);
            for (int j = 0; j < nb && ok; ++j)
                for (int h = 0; h < H && ok; ++h) ok = push(&tm_k, h * N + j * 128, SLOT);
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            uint32_t ring_tail = 0, ph_pe = 0, ph_qc = 0, ph_p[2] = {0, 0};
            bool ok = true;
            auto consume = [&](int& slot) -> bool {
                slot = ring_tail % NS;
                uint32_t ph = (ring_tail / NS) & 1;
                if (!W.wait(&sh.full[slot], ph, 81)) return false;
                tc_fence_after();
                ++ring_tail;
                return true;
            };
            // S_i for i = j H + h (key block j, head h) into buffer i mod 2
            auto issue_s = [&](int i, int h) -> bool {
                int sl;
                if (!consume(sl)) return false;
                const uint64_t db = desc_sw128(s_ring + sl * SLOT);
                const uint32_t sd = tmem + T_S0 + 128 * (i & 1);
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(sd, tmem + T_QP + 32 * h + 8 * kk, db + 2 * kk, idesc_bf16(128, 128, false), kk > 0);
                mma_commit(smem_u32(&sh.empty[sl]));
                mma_commit(smem_u32(&sh.bar_s[i & 1]));
                return true;
            };
            for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
                if (!(ok = W.wait(&sh.bar_pe, ph_pe, 82))) break;
                tc_fence_after();
                // Q projections, QROUND heads at a time into the S buffers' columns
                for (int h0 = 0; h0 < H && ok; h0 += QROUND) {
                    for (int h = h0; h < H && h < h0 + QROUND && ok; ++h) {
                        int slot;
                        if (!(ok = consume(slot))) break;
                        const uint64_t da = desc_sw128(s_pe), db = desc_sw128(s_ring + slot * SLOT);
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss(tmem + T_QA + 64 * (h - h0), da + 2 * kk, db + 2 * kk, idesc_bf16(128, 64, false),
                                   kk > 0);
                        mma_commit(smem_u32(&sh.empty[slot]));
                    }
                    if (!ok) break;
                    mma_commit(smem_u32(&sh.bar_q));
                    // packed (and the accumulators read) before the next round or the first S overwrites them
                    if (!(ok = W.wait(&sh.bar_qc, ph_qc, 83))) break;
                    tc_fence_after();
                }
                if (!ok) break;
                const int n_s = nb * H;
                int hi = 0;   // head of the next S to issue
                for (int i = 0; i < n_s && i < 2 && ok; ++i) {
                    ok = issue_s(i, hi);
                    if (++hi == H) hi = 0;
                }
                for (int i = 0; i < n_s && ok; ++i) {
                    if (!(ok = W.wait(&sh.bar_p[i & 1], ph_p[i & 1], 84))) break;
                    tc_fence_after();
                    if (i + 2 < n_s) {
                        ok = issue_s(i + 2, hi);
                        if (++hi == H) hi = 0;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ compute
        const int wg = tid >> 7, row = tid & 127;
        const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        uint32_t ph_q = 0, ph_s[2] = {0, 0}, ph_cs = 0;
        const float qscale = 0.125f * kLog2e;
        bool ok = true;
        auto arrive = [&](uint64_t* b) { mbar_arrive(smem_u32(b)); };
        auto csync = [&](int site) -> bool {
            arrive(&sh.bar_cs);
            return W.wait(&sh.bar_cs, ph_cs, site);
        };
        const int my_slot = row / np;            // sub-volume slot of this row
        const int my_i = row % np;               // probe index within it
        const int warps_per_tile = np >= 32 ? np / 32 : 1;   // per warpgroup
        for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
            const int t_idx = unit * tpu + my_slot;
            const bool valid = my_slot < tpu && t_idx < n_sel;
            const int t = valid ? a.sel_tiles[t_idx] : -1;
            float p[3] = {0.f, 0.f, 0.f};
            bool has_probe = valid;   // this row holds a probe of sub-volume t
            if (valid && a.probe_xyz) {
                const int beg = a.probe_off[t];
                has_probe = my_i < a.probe_off[t + 1] - beg;
                if (has_probe) {
                    p[0] = a.probe_xyz[3 * (size_t)(beg + my_i)];
                    p[1] = a.probe_xyz[3 * (size_t)(beg + my_i) + 1];
                    p[2] = a.probe_xyz[3 * (size_t)(beg + my_i) + 2];
                }
            } else if (valid) {
                const int e = a.qorder[8 * a.tile_off[t] + my_i];
                voxel_point(child_index(a.plist[e >> 3], e & 7, a.R), a.R, p);
            }
            for (int c = 2 * wg; c < 2 * wg + 2; ++c) {
                uint32_t w[4];
                for (int v = 0; v < 4; ++v) w[v] = pack_bf16(pe_lane(p, c * 8 + 2 * v), pe_lane(p, c * 8 + 2 * v + 1));
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(swz(s_pe, row, c)), "r"(w[0]),
                             "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
            }
            fence_proxy_async();
            arrive(&sh.bar_pe);
            const float* ml = has_probe ? a.probe_ml + ((size_t)t * np + my_i) * H * 2 : nullptr;
            // Q of every head: + bq, scale, bf16 pairs; warpgroup g packs head dims [16g, 16g+16) into
            // columns [32h + 8g, 32h + 8g + 8)
            for (int h0 = 0; h0 < H && ok; h0 += QROUND) {
                if (!(ok = W.wait(&sh.bar_q, ph_q, 86))) break;
                tc_fence_after();
                for (int h = h0; h < H && h < h0 + QROUND; ++h) {
                    float q[16];
                    tmem_ld16(trow + T_QA + 64 * (h - h0) + 16 * wg, q);
                    tmem_wait_ld();
                    reg_fence16(q);
                    uint32_t pk[8];
                    for (int v = 0; v < 8; ++v) {
                        const int c0 = h * 64 + 16 * wg + 2 * v;
                        pk[v] = pack_bf16((q[2 * v] + a.bq[c0]) * qscale, (q[2 * v + 1] + a.bq[c0 + 1]) * qscale);
                    }
                    tmem_st8(trow + T_QP + 32 * h + 8 * wg, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                arrive(&sh.bar_qc);
            }
            int pb = 0;   // partial-sum buffer
            int i = 0;    // S index: key block j, head h -> i = j H + h
            // A column of a sub-volume sums the partials of the warps that hold its rows in the
            // column's warpgroup: one warp (32 probes) or two (64), added straight into the score
            // row (a shared-memory atomic add of two terms onto zero gives the same value in
            // either order), so no barrier per key block; four (128) go through the partial
            // buffer in a fixed order.
            const bool direct = warps_per_tile <= 2;
            const int my_sv = (32 * (warp & 3)) / np;
            if (direct && warps_per_tile == 2) {
                for (int idx = tid; idx < tpu * N; idx += NCOMP) score[idx] = 0.f;
                if (!(ok = csync(97))) break;
            }
            for (int j = 0; j < nb && ok; ++j) {
                const int vcols = N - j * 128 - 32 * wg;   // own columns < vcols are real tokens
                float acc[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) acc[c] = 0.f;
                for (int h = 0; h < H; ++h, ++i) {
                    if (!(ok = W.wait(&sh.bar_s[i & 1], ph_s[i & 1], 87))) break;
                    tc_fence_after();
                    const uint32_t sb = trow + T_S0 + 128 * (i & 1) + 32 * wg;
                    // P = 2^(S - m) / l = 2^(S - m - log2 l); rows without a probe add 2^-inf = 0
                    const float mo = has_probe ? ml[h * 2] + __log2f(ml[h * 2 + 1]) : INFINITY;
                    float s0[32];
                    tmem_ld32(sb, s0);
                    tmem_wait_ld();
                    reg_fence(s0);
                    tc_fence_before();
                    arrive(&sh.bar_p[i & 1]);   // this quarter of S_i consumed
                    if (vcols >= 32) {
                        const uint64_t mm = f32x2(mo, mo);
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            float d0, d1, a0, a1;
                            f32x2_split(sub_f32x2(f32x2(s0[c], s0[c + 1]), mm), d0, d1);
                            f32x2_split(add_f32x2(f32x2(acc[c], acc[c + 1]), f32x2(ex2(d0), ex2(d1))), a0, a1);
                            acc[c] = a0;
                            acc[c + 1] = a1;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) acc[c] += c < vcols ? ex2(s0[c] - mo) : 0.f;
                    }
                }
                if (!ok) break;
                const float cs = warp_colsum32(acc, lane);
                if (direct) {
                    const int col = j * 128 + 32 * wg + lane;
                    if (col < N) {
                        float* dst = score + (size_t)my_sv * N + col;
                        if (warps_per_tile == 1) *dst = cs;
                        else atomicAdd(dst, cs);
                    }
                    continue;
                }
                part[(pb * 16 + warp) * 32 + lane] = cs;
                if (!(ok = csync(88))) break;
                // column col of sub-volume s: its warps of the column's warpgroup, in order
                for (int idx = tid; idx < tpu * 128; idx += NCOMP) {
                    const int sv = idx >> 7, col = idx & 127;
                    if (j * 128 + col < N) {
                        const int g = col >> 5;
                        const float* pp = part + (pb * 16 + 4 * g + sv * warps_per_tile) * 32 + (col & 31);
                        float sum = 0.f;
                        for (int w = 0; w < warps_per_tile; ++w) sum += pp[w * 32];
                        score[(size_t)sv * N + j * 128 + col] = sum;
                    }
                }
                pb ^= 1;
            }
            if (!ok) break;
            if (!(ok = csync(89))) break;
            if (a.score_out) {   // debug export of the unit's score rows
                for (int idx = tid; idx < tpu * N; idx += NCOMP) {
                    const int sv = idx / N;
                    if (unit * tpu + sv < n_sel) {
                        const int ts = a.sel_tiles[unit * tpu + sv];
                        if (ts < a.score_rows) a.score_out[(size_t)ts * N + (idx - sv * N)] = score[idx];
                    }
                }
            }
            // ------------------------------------------------ Top-K per sub-volume
            const int k = a.top_k;
            for (int s = 0; s < tpu && ok; ++s) {
                const int ti = unit * tpu + s;
                if (ti >= n_sel) break;
                const int t_s = a.sel_tiles[ti];
                const float* sc = score + (size_t)s * N;
                int32_t* out = a.sel + (size_t)t_s * k;
                if (k >= N) {
                    for (int j = tid; j < N; j += NCOMP) out[j] = j;
                    continue;
                }
                uint32_t prefix = 0, pmask = 0;
                int need = k;
                for (int shift = 24; shift >= 0 && ok; shift -= 8) {
                    for (int b = tid; b < 256; b += NCOMP) sh.hist[b] = 0;
                    if (!(ok = csync(90))) break;
                    for (int j = tid; j < N; j += NCOMP) {
                        const uint32_t key = __float_as_uint(sc[j]);
                        if ((key & pmask) == prefix) atomicAdd(&sh.hist[(key >> shift) & 255], 1);
                    }
                    if (!(ok = csync(91))) break;
                    if (tid == 0) {
                        int acc = 0, b = 255;
                        for (; b > 0; --b) {
                            if (acc + sh.hist[b] >= need) break;
                            acc += sh.hist[b];
                        }
                        sh.red[0] = b;
                        sh.red[1] = need - acc;
                    }
                    if (!(ok = csync(92))) break;
                    prefix |= (uint32_t)sh.red[0] << shift;
                    pmask |= 255u << shift;
                    need = sh.red[1];
                }
                if (!ok) break;
                const uint32_t thr = prefix;
                const int per = (N + NCOMP - 1) / NCOMP;
                const int j_lo = tid * per, j_hi = min(N, j_lo + per);
                int eq = 0;
                for (int j = j_lo; j < j_hi; ++j) eq += __float_as_uint(sc[j]) == thr;
                int x = eq;
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                if (lane == 31) sh.wsum[warp] = x;
                if (!(ok = csync(93))) break;
                int eq_before = x - eq;
                for (int w = 0; w < warp; ++w) eq_before += sh.wsum[w];
                if (!(ok = csync(94))) break;
                int take = 0;
                {
                    int e = eq_before;
                    for (int j = j_lo; j < j_hi; ++j) {
                        const uint32_t key = __float_as_uint(sc[j]);
                        take += key > thr || (key == thr && e < need);
                        e += key == thr;
                    }
                }
                x = take;
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                if (lane == 31) sh.wsum[warp] = x;
                if (!(ok = csync(95))) break;
                int pos = x - take;
                for (int w = 0; w < warp; ++w) pos += sh.wsum[w];
                {
                    int e = eq_before;
                    for (int j = j_lo; j < j_hi; ++j) {
                        const uint32_t key = __float_as_uint(sc[j]);
                        if (key > thr || (key == thr && e < need)) out[pos++] = j;
                        e += key == thr;
                    }
                }
                if (!(ok = csync(96))) break;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// Probes given as points: probe p of tile t (p in [probe_off[t], probe_off[t+1])) keeps its
// softmax statistics in row t * n_probe + (p - probe_off[t]); every tile is scored.
__global__ void flat_probe_slots_kernel(const int32_t* __restrict__ probe_off, int T, int n_probe,
                                        int32_t* __restrict__ ml_slot, int32_t* __restrict__ sel_tiles,
                                        int32_t* __restrict__ n_sel) {
    const int warps = gridDim.x * (blockDim.x >> 5);
    const int lane = threadIdx.x & 31;
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
        const int beg = probe_off[t], end = probe_off[t + 1];
        for (int p = beg + lane; p < end; p += 32) ml_slot[p] = t * n_probe + (p - beg);
        if (lane == 0) sel_tiles[t] = t;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *n_sel = T;
}

}  // namespace

vdm_status launch_flat_probe_slots(const int32_t* probe_off, int T, int n_probe, int32_t* ml_slot,
                                   int32_t* sel_tiles, int32_t* n_sel, cudaStream_t s) {
    if (T <= 0) return VDM_OK;
    const int grid = (T + 7) / 8 < 1184 ? (T + 7) / 8 : 1184;
    flat_probe_slots_kernel<<<grid, 256, 0, s>>>(probe_off, T, n_probe, ml_slot, sel_tiles, n_sel);
    return check_launch("flat_probe_slots_kernel");
}

static size_t select_tc_smem(int n_probe, int N) {
    return 1024 + 16384 + (size_t)NS * SLOT + (size_t)(128 / n_probe) * N * 4 + 2 * 4 * 128 * 4;
}

bool select_tc_supported(int C, int n_probe, int N, vdm_dtype dt) {
    return dt == VDM_BF16 && (C == 128 || C == 256 || C == 512) && (n_probe == 32 || n_probe == 64 || n_probe == 128) &&
           select_tc_smem(n_probe, N) <= 227 * 1024;
}

vdm_status launch_select_tc(const SelectTcLaunch& L, cudaStream_t st) {
    if (L.T <= 0) return VDM_OK;
    SelArgs a;
    a.C = L.C; a.H = L.H; a.N = L.N;
    a.bq_unused = nullptr;
    a.bq = L.bq;
    a.n_sel_max = L.T;
    a.n_sel = L.n_sel;
    a.sel_tiles = L.sel_tiles;
    a.tile_off = L.tile_off;
    a.plist = L.plist;
    a.qorder = L.qorder;
    a.probe_xyz = L.probe_xyz;
    a.probe_off = L.probe_off;
    a.probe_ml = L.probe_ml;
    a.R = L.R;
    a.n_probe = L.n_probe;
    a.tpu = 128 / L.n_probe;
    a.top_k = L.top_k;
    a.sel = L.sel;
    a.score_out = L.score_out;
    a.score_rows = L.score_rows;
    a.err = tc_error_word();
    if (!a.err) return fail(VDM_ERR_CUDA, "error word lookup failed");
    a.timeout = 4000000000ll;
    CUtensorMap m_wq64, m_k;
    VDM_TRY(make_bf16_map(&m_wq64, L.Wq, L.C, 64, 64, 64));
    VDM_TRY(make_bf16_map(&m_k, L.K, (int64_t)L.H * L.N, 64, 128, 64));
    const size_t smem = select_tc_smem(L.n_probe, L.N);
    if (smem > 227 * 1024) return fail(VDM_ERR_UNSUPPORTED, "selection needs %zu bytes of shared memory", smem);
    cudaError_t e = cudaFuncSetAttribute(select_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "select_tc smem attribute: %s", cudaGetErrorString(e));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int max_units = (L.T + a.tpu - 1) / a.tpu;
    const int grid = max_units < sms ? max_units : sms;
    prof_begin(kProfSelect, st);
    select_tc_kernel<<<grid, NT, smem, st>>>(m_wq64, m_k, a);
    prof_end(kProfSelect, st);
    return check_launch("select_tc_kernel");
}

}  // namespace vdm
