// Fused vecset decoder on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// The decoder of FlashVDM ("Unleashing Vecset Diffusion Model for Fast Shape
// Generation", aipaper.cc summary, section 3: cross-attention from query
// points to the latent set, then the SDF; section 4.1 item 2: attention over
// a per-sub-volume token subset) for bf16 weights and K/V, fp32 accumulation.
// One persistent CTA per SM decodes 128-query tiles; nothing but the final
// SDF value (and, for probe queries, their softmax statistics) leaves the SM.
//
// Warp roles (384 threads; 320 for CTA pairs):
//   warps 0-7  compute: two warpgroups; thread (g, r) owns TMEM lane r and
//              half g of the row's columns (head dims, hidden units, LayerNorm
//              columns), so every SM sub-partition runs two compute warps; in
//              the attention warpgroup g owns the key blocks j = g mod 2 and
//              runs its own online softmax over them (own maximum, sum and O
//              accumulator); the two combine once per head;
//   warp 8     MMA issue (the whole warp runs the loop; one elected lane issues);
//   warp 9     producer: TMA loads of weights and of contiguous K/V blocks,
//              cp.async gathers of a sub-volume's selected K/V rows (each lane's
//              copies arrive on the slot's barrier when they land);
//   warp 10    (single CTAs) the attention's P V MMAs, from a ring of values of
//              their own, so that block j's P V and the S of block j+3 (which
//              waits for that P V to have read P_j) are issued by different
//              warps and the issue chain of one block no longer holds the next;
//   warp 11    (single CTAs) the values' producer (TMA or gathers), so that the
//              value ring refills without waiting behind the other ring;
// connected only by mbarriers (no CTA-wide barrier inside a tile).
// Compiled twice per width: one CTA per 128-row MMA, or (cta_group::2) a CTA
// pair of a cluster per 256-row MMA, each CTA holding half of every B tile.
//
// Split-packed A operand: the GELU output is produced by the two warpgroups,
// each packing its half (bf16 pairs) into the start of its own fp32 source
// columns (so neither overwrites the other's unread source); the k-step q of
// 16 elements then sits at column  g*W/2 + (16q mod W/2)/2  with g = 16q / (W/2)
// for a W-wide block.  The softmax probabilities P_j are packed in place, each
// 32-column chunk's bf16 pairs in the chunk's first 16 columns.
//
// Per tile:
//   PE (bf16 smem) ; per head h: Q_h = PE Wq_h^T (fp32 in TMEM) -> + bq, scaled,
//   bf16 in smem (attention-output atom h, free until the head's combine);
//   per 128-token block j, owned by warpgroup g = j mod 2: S_j = Q_h K_j^T into
//   S_{j mod 3} ; softmax of the block -> P_j (bf16, in place) ; O_g += P_j V_j ;
//   end of head: combine the two (max, sum, O_g) -> a[:, h] (bf16 smem).
//   (Single CTAs project Q for every head at the start of the tile and run the
//   blocks of all heads as one stream b = h nb + j, S_b in S_{b mod 3}, so the
//   next head's scores are computed during a head's combine.)
//   X = PE Wq^T + a Wo^T ; LN1 -> bf16 smem ; MLP hidden chunks:
//   H_c = LN1(x1) W1_c^T, GELU, X += GELU(H_c) W2_c^T ; LN2 . w_head -> SDF.
//
// TMEM (512 columns x 128 lanes):
//   attention: S0 [0,128) S1 [128,256) S2 [256,384) (P_j overwrites the first 16 of
//              each 32 S columns once they are read; CTA pairs accumulate Q_h in S2
//              before the head's first block, single CTAs every head's Q in [0, C)
//              at the start of the tile) O0 [384,448) O1 [448,512)
//   output projection: X [0, C)
//   MLP, C <= 256: acc [0, C); hidden chunks (128 wide) at [256,384) [384,512)
//   MLP, C == 512: the 128 x 512 fp32 residual alone fills TMEM, so the MLP
//              output is produced in two 256-wide halves (the hidden projection
//              is recomputed for the second half); while the first half runs,
//              x1's second half (fp32) waits in a per-CTA global parking area
//              (L2 resident); hidden chunks (128 wide) at [256,384) [384,512).
//
// Softmax: logits in log2 units (the 1/8 scale and log2 e folded into Q);
// the running maximum is only raised when a block exceeds it by more than 8
// (then O and the sum are rescaled), so P stays <= 2^8.  A quarter of the
// exponentials run on the FMA pipe (exp2_pair_poly), the rest on ex2.approx.
//
// Barrier protocol: waits are parity based, so every waiter observes every
// phase of the barriers it uses, and no barrier can run two phases ahead of a
// waiter (each producer step depends on the waiter's previous step).
// Every wait on an mbarrier is bounded: on expiry the kernel records the site
// in an error word, flags the CTA and winds down.
#include <cuda.h>
#include <stdio.h>
#include <string.h>

#include "tc_ptx.cuh"
#include "vdm_internal.cuh"

namespace vdm {

namespace {

using namespace ptx;

constexpr int BM = 128;        // queries per tile (TMEM lanes)
constexpr int NCOMP = 256;     // compute threads (two warpgroups)
constexpr int NT = 320;        // + MMA warp + producer warp (CTA pairs)
constexpr int NT_SPLIT = 384;  // single CTAs: + a P V issue warp and a value producer warp
constexpr int WARP_MMA = 8, WARP_PROD = 9, WARP_PV = 10, WARP_VPROD = 11;
constexpr int SLOT = 16384;    // ring slot bytes
constexpr int MAX_NS = 16;   // ring slots (CTA pairs use twice as many, half as large)
constexpr int RING_ARRIVALS = 32;   // arrivals completing a ring slot: one per producer lane
constexpr float kLog2e = 1.4426950408889634f;

// attention: three S buffers in rotation (block j in S_{j mod 3}; its P overwrites the S
// columns already read), so the next block's scores are ready before a warpgroup needs them;
// the warpgroups alternate blocks, so one's exponentials overlap the other's loads, maximum
// and hand-offs; one O accumulator per warpgroup (its blocks, all 64 head dims); the packed
// Q of a head waits in shared memory
#ifndef VDM_EMU_PAIRS
#define VDM_EMU_PAIRS 0x8888u
#endif
// Column pairs (bit v: columns 2v, 2v+1 of every 32) whose softmax exponentials run on the
// FMA pipe (exp2_pair_poly) instead of the special-function unit.
constexpr uint32_t kEmuPairs = VDM_EMU_PAIRS;
constexpr uint32_t T_S0 = 0, T_O0 = 384, T_O1 = 448, T_QACC = 256;
constexpr int NSB = 3;   // S buffers

// ring depth: 16 KB slots in what the 227 KB of shared memory leaves after the
// activation buffer (C/64 atoms of 16 KB), the embedding tile and alignment
__host__ __device__ constexpr int ring_slots(int C) {
    return (int)((227 * 1024 - ((C / 64) * 16384 + 16384 + 1024) - 512) / SLOT) < MAX_NS / 2
               ? (int)((227 * 1024 - ((C / 64) * 16384 + 16384 + 1024) - 512) / SLOT)
               : MAX_NS / 2;
}

struct TcArgs {
    DecodeArgs d;
    int ns;
    float* park;         // C == 512: per-CTA parking area, 128 x 256 fp32 each
    int* err;
    long long timeout;   // cycles per bounded wait
    int inject;          // test hook: withhold the first Q-projection completion signal
};

struct Shared {
    uint64_t full[MAX_NS], empty[MAX_NS];
    // MMA commits (count 1); bar_hd and bar_w2 are waited on by the MMA warp only
    // bar_s[j mod 6]: S_j ready (block j's buffer and owner both follow from j mod 6)
    // bar_pvm[e mod 3]: the e-th P V product that an S issue waits for is complete
    uint64_t bar_q, bar_s[6], bar_pvg[2], bar_pvm[3], bar_pv, bar_x, bar_h[2], bar_acc, bar_hd, bar_w2, bar_fin,
        bar_fin2;
    // compute-warp arrivals (count 128)
    // bar_cmb (single CTAs): a head's combine has read O0 and O1 (the next head's first P V may overwrite them)
    uint64_t bar_pe, bar_qc, bar_p[2], bar_a, bar_hin, bar_r, bar_g[2], bar_cs, bar_wg, bar_cmb;
    uint32_t tmem_base;
    int abort;
    float G, Bc;     // SDF head folded with LN2's affine: sum w g, sum w b + b_head
    float Gt, Bt;    // the same for the tSDF head
};

struct Waiter {
    Shared* sh;
    int* err;
    long long timeout;
    uint32_t peer_abort;   // CTA pairs: shared::cluster address of the other CTA's abort flag (else 0)
    bool cluster_acq;      // acquire at cluster scope (barriers that collect the other CTA's arrivals)
    // Wait for the phase with parity `phase` to complete; flips `phase`.  Called by
    // whole warps (every role runs converged); the result is the same in all lanes.
    __device__ bool wait(uint64_t* bar, uint32_t& phase, int site) {
        const uint32_t b = smem_u32(bar);
        long long t0 = 0;
        bool done = false;
        for (uint32_t it = 0;; ++it) {
            if (cluster_acq ? mbar_try_wait_cluster(b, phase) : mbar_try_wait(b, phase)) {
                phase ^= 1;
                done = true;
                break;
            }
            if ((it & 63) == 63) {
                if (*reinterpret_cast<volatile int*>(&sh->abort)) break;
                const long long t = clock64();
                if (t0 == 0) t0 = t;
                else if (t - t0 > timeout) {
                    *reinterpret_cast<volatile int*>(&sh->abort) = 1;
                    if (peer_abort) st_cluster_u32(peer_abort, 1u);
                    atomicCAS(err, 0, site);
                    break;
                }
            }
        }
        return __all_sync(0xffffffffu, done);
    }
};

// Wind-down wait for our own asynchronous work (loads, MMAs), which always
// completes; bounded by `cycles` all the same, and not cut short by an abort.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, long long cycles) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity) && clock64() - t0 < cycles) {
    }
}

__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int c) {
    return base + r * 128 + ((c ^ (r & 7)) << 4);
}
// 64-byte rows, 64 B swizzle: the 16-byte chunk index is XORed with address bits 7-8
__device__ __forceinline__ uint32_t swz64(uint32_t base, int r, int c) {
    return base + r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

// TMEM column of k-step q (16 elements) of a W-wide split-packed A operand
__device__ __forceinline__ uint32_t split_col(int q, int W) {
    const int half = W / 2, g0 = 16 * q;
    return (uint32_t)((g0 / half) * half + (g0 % half) / 2);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t* w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3])
                 : "memory");
}

// Work unit -> queries (identical in every role).
struct Unit {
    int nq;
    int64_t qbeg;        // first query slot
    int t;               // tile (tile modes)
    int first;           // first position inside the tile's dense / sparse range
    const int32_t* sel;  // selected tokens (sparse mode)
};

__device__ __forceinline__ Unit unit_of(const DecodeArgs& a, int64_t unit) {
    Unit u;
    u.sel = nullptr;
    u.t = -1;
    u.first = 0;
    if (a.work == kWorkFlat) {
        const int64_t M = a.M_dev ? (int64_t)*a.M_dev : a.M;
        u.qbeg = unit * BM;
        u.nq = u.qbeg < M ? (int)(M - u.qbeg < BM ? M - u.qbeg : BM) : 0;
        return u;
    }
    // slot-major order: units t, t + T, ... of one sub-volume are a grid stride apart, so the
    // persistent CTAs' static round-robin deals every slot index to every CTA (a tile-major
    // order with T * slots units would give CTA c only slot c mod slots, and the later slots
    // of a sub-volume are often empty)
    const int t = (int)(unit % a.T), sl = (int)(unit / a.T);
    const int cnt = 8 * (a.tile_off[t + 1] - a.tile_off[t]);
    int lo, n;
    if (a.work == kWorkTileDense) {
        lo = 0;
        n = cnt < a.n_probe ? cnt : a.n_probe;
    } else {
        lo = a.n_probe;
        n = cnt > a.n_probe ? cnt - a.n_probe : 0;
        u.sel = a.sel + (size_t)t * a.ksel;
    }
    const int first = lo + sl * BM;
    u.nq = first < lo + n ? min(BM, lo + n - first) : 0;
    u.qbeg = 8 * (int64_t)a.tile_off[t] + first;
    u.t = t;
    u.first = first;
    return u;
}

// ---------------------------------------------------------------- the kernel
template <int CC, int CG>
__global__ void __launch_bounds__(CG == 2 ? NT : NT_SPLIT, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_wq, const __grid_constant__ CUtensorMap tm_wq64,
                 const __grid_constant__ CUtensorMap tm_wo, const __grid_constant__ CUtensorMap tm_w1,
                 const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const TcArgs ta) {
    const DecodeArgs& a = ta.d;
    extern __shared__ uint8_t dyn_raw[];
    __shared__ Shared sh;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // the model width fixes the TMEM plan, the ring depth and every MMA shape at compile time
    constexpr int C = CC;
    const int H = a.H, F = a.F, N = a.N;
    constexpr int NA = C / 64;
    constexpr bool halves = C > 256;
    constexpr int HN = 128;
    constexpr int NS = ring_slots(C);   // 16 KB slots that fit
    constexpr int CW = halves ? 256 : C;
    constexpr int n_half = halves ? 2 : 1;
    constexpr uint32_t T_H0 = 256, T_H1 = 384;
    const int n_chunks = F / HN;
    constexpr int w1_gran = NA;
    constexpr int w2_gran = (CW / 128) * (HN / 64);
    // CG == 2: the CTA pair of a cluster runs 256-row MMAs; each CTA loads half of
    // every B operand (its N/2 rows), the even CTA issues the MMAs, and the odd
    // CTA forwards the completion of its loads to the even CTA's ring barriers.
    constexpr bool PAIR = CG == 2;
    const uint32_t crank = PAIR ? cluster_rank() : 0u;
    const bool leader = crank == 0;
    constexpr int BR = PAIR ? 64 : 128;   // weight / key rows of a 128-row B tile held by this CTA
    // ring items: a CTA of a pair holds half of each weight tile (8 KB), so one 16 KB slot
    // carries two consecutive 64-wide K atoms (8 MMA k-steps per wait and release)
    constexpr int RS = SLOT;
    constexpr int NR = NS;
    // Single CTAs split the MMA issue over two warps: the P V products of the attention run on
    // WARP_PV, everything else on WARP_MMA, so a block's P V and the S of a later block are issued
    // side by side.  The values then travel in a ring of their own (slots NRA..NR-1, consumed by
    // WARP_PV), the other items in slots 0..NRA-1 (consumed by WARP_MMA); each ring has one
    // producer and one consumer in FIFO order.
    constexpr bool SPLIT = !PAIR;
    constexpr int NRB = SPLIT ? 2 : 0;
    constexpr int NRA = NR - NRB;
    static_assert(NRA >= 2, "ring too small");
    constexpr int AT = PAIR ? 2 : 1;      // K atoms per weight item
    constexpr int KA = NA + 1;            // output-projection K atoms: embedding + attention

    const uint32_t dyn0 = (smem_u32(dyn_raw) + 1023u) & ~1023u;
    const uint32_t s_abuf = dyn0;
    const uint32_t s_pe = s_abuf + NA * 16384;
    const uint32_t s_ring = s_pe + 16384;

    Waiter W{&sh, ta.err, ta.timeout, PAIR ? mapa(smem_u32(&sh.abort), crank ^ 1u) : 0u, false};

    if (tid == 0) {
        for (int i = 0; i < NR; ++i) {
            // a slot is complete when the producer warp's 32 lanes arrived (a TMA item: one counted
            // arrival plus its bytes; a gathered item: each lane once its copies landed) and, in the
            // even CTA of a pair, the odd CTA's forward
            mbar_init(smem_u32(&sh.full[i]), RING_ARRIVALS + (PAIR && leader ? 1 : 0));
            mbar_init(smem_u32(&sh.empty[i]), 1);
        }
        uint64_t* one[] = {&sh.bar_q, &sh.bar_s[0], &sh.bar_s[1], &sh.bar_s[2], &sh.bar_s[3], &sh.bar_s[4],
                           &sh.bar_s[5], &sh.bar_pvg[0], &sh.bar_pvg[1], &sh.bar_pvm[0], &sh.bar_pvm[1],
                           &sh.bar_pvm[2], &sh.bar_pv, &sh.bar_x, &sh.bar_h[0], &sh.bar_h[1], &sh.bar_acc,
                           &sh.bar_hd, &sh.bar_w2, &sh.bar_fin, &sh.bar_fin2};
        for (auto* b : one) mbar_init(smem_u32(b), 1);
        // compute -> MMA: one arrival per compute thread, or per compute warp of both CTAs
        uint64_t* to_mma[] = {&sh.bar_pe, &sh.bar_qc, &sh.bar_a,
                              &sh.bar_hin, &sh.bar_r, &sh.bar_g[0], &sh.bar_g[1]};
        for (auto* b : to_mma) mbar_init(smem_u32(b), PAIR ? 2 * (NCOMP / 32) : NCOMP);
        // P_j comes from one warpgroup (the one that owns block j)
        for (auto* b : {&sh.bar_p[0], &sh.bar_p[1]}) mbar_init(smem_u32(b), PAIR ? 2 * (BM / 32) : BM);
        mbar_init(smem_u32(&sh.bar_cs), NCOMP);
        mbar_init(smem_u32(&sh.bar_wg), NCOMP);
        mbar_init(smem_u32(&sh.bar_cmb), NCOMP);
        sh.abort = 0;
        fence_mbar_init();
        fence_proxy_async();
    }
    if (warp == 1) {
        float g = 0.f, bc = 0.f, gt = 0.f, bt = 0.f;
        for (int c = lane; c < C; c += 32) {
            const float w = a.w_head[c];
            g += a.query_ln ? w * a.ln2_g[c] : w;
            bc += a.query_ln ? w * a.ln2_b[c] : 0.f;
            if (a.w_tsdf) {
                const float wt = a.w_tsdf[c];
                gt += a.query_ln ? wt * a.ln2_g[c] : wt;
                bt += a.query_ln ? wt * a.ln2_b[c] : 0.f;
            }
        }
        for (int o = 16; o; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            bc += __shfl_xor_sync(0xffffffffu, bc, o);
            gt += __shfl_xor_sync(0xffffffffu, gt, o);
            bt += __shfl_xor_sync(0xffffffffu, bt, o);
        }
        if (lane == 0) {
            sh.G = g;
            sh.Bc = bc + a.b_head[0];
            sh.Gt = gt;
            sh.Bt = a.w_tsdf ? bt + a.b_tsdf[0] : 0.f;
        }
    }
    if (warp == 0) {
        if (PAIR) {
            tmem_alloc_pair(smem_u32(&sh.tmem_base), 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(&sh.tmem_base), 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();   // both CTAs' barriers are initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    // Work: units of 128 queries; a CTA pair takes two units that attend to the same keys
    // (consecutive flat units, or two slots of one sub-volume) and skips a pair only when
    // both are empty.
    // single CTAs in the sparse pass take the non-empty units from a list (equal shares per CTA)
    const bool listed = !PAIR && a.work == kWorkTileSparse && a.unit_list != nullptr;
    const int64_t n_units = a.work == kWorkFlat ? (a.M + BM - 1) / BM
                            : listed             ? (int64_t)*a.n_units_dev
                                                 : (int64_t)a.T * a.slots;
    const int spt = PAIR ? (a.slots + 1) / 2 : a.slots;   // slot pairs per sub-volume
    const int64_t n_iter = !PAIR ? n_units : a.work == kWorkFlat ? (n_units + 1) / 2 : (int64_t)a.T * spt;
    const int64_t it0 = PAIR ? blockIdx.x / 2 : blockIdx.x;
    const int64_t it_step = PAIR ? gridDim.x / 2 : gridDim.x;
    auto unit_at = [&](int64_t it, uint32_t r) -> Unit {
        if (!PAIR) return unit_of(a, listed ? (int64_t)a.unit_list[it] : it);
        if (a.work == kWorkFlat) return unit_of(a, 2 * it + r);
        const int64_t t = it % a.T;
        const int sl = 2 * (int)(it / a.T) + (int)r;
        if (sl < a.slots) return unit_of(a, (int64_t)sl * a.T + t);
        Unit u = unit_of(a, t);   // same sub-volume (same keys), no queries
        u.nq = 0;
        return u;
    };
    auto active = [&](int64_t it) -> bool {
        if (unit_at(it, crank).nq > 0) return true;
        return PAIR && unit_at(it, crank ^ 1u).nq > 0;
    };
    // barriers of the MMA-issuing CTA, and commits that reach both CTAs
    auto lead_bar = [&](uint64_t* b) -> uint32_t { return PAIR ? mapa(smem_u32(b), 0u) : smem_u32(b); };
    // (issued by the whole MMA warp; one elected lane commits)
    auto commit_both = [&](uint64_t* b) {
        if (PAIR) {
            mma_commit_pair_w(mapa(smem_u32(b), 0u));
            mma_commit_pair_w(mapa(smem_u32(b), 1u));
        } else {
            mma_commit_w(smem_u32(b));
        }
    };
    auto commit_own = [&](uint64_t* b) {
        if (PAIR) mma_commit_pair_w(smem_u32(b));
        else mma_commit_w(smem_u32(b));
    };
    // items a unit pushes through the ring (producer, MMA and forwarder agree on it)
    auto n_items = [&](int nb) -> int {
        return H * (1 + 2 * nb) + (C / 128) * ((KA + AT - 1) / AT) +
               n_half * n_chunks * (w1_gran / AT + w2_gran / AT);
    };

    // ==================================================================== producer
    if (warp == WARP_PROD || (SPLIT && warp == WARP_VPROD)) {
        // single CTAs: WARP_PROD fills ring A (weights, keys), WARP_VPROD ring B (values)
        const bool vprod = SPLIT && warp == WARP_VPROD;
        uint32_t head_a = 0, head_b = 0;   // items pushed into each ring
        const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(a.K);
        const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.V);
        bool ok = true;
        int pa_slot = 0, pb_slot = 0;
        uint32_t pa_ph = 1, pb_ph = 1;   // parity of the empty-phase a reused slot waits for (first pass: none)
        // ring B (values, single CTAs) when `vring`, else ring A
        auto take_slot = [&](int& slot, bool vring) -> bool {
            if constexpr (NRB > 0) {
                if (vring) {
                    slot = NRA + pb_slot;
                    if (head_b >= (uint32_t)NRB) {
                        uint32_t ph = pb_ph;
                        if (!W.wait(&sh.empty[slot], ph, 41)) return false;
                    }
                    ++head_b;
                    if (++pb_slot == NRB) {
                        pb_slot = 0;
                        pb_ph ^= 1;
                    }
                    return true;
                }
            }
            slot = pa_slot;
            if (head_a >= (uint32_t)NRA) {
                uint32_t ph = pa_ph;
                if (!W.wait(&sh.empty[slot], ph, 40)) return false;
            }
            ++head_a;
            if (++pa_slot == NRA) {
                pa_slot = 0;
                pa_ph ^= 1;
            }
            return true;
        };
        auto push_tma = [&](const CUtensorMap* m, int x, int y, uint32_t bytes, bool vring = false) -> bool {
            int slot;
            if (!take_slot(slot, vring)) return false;
            if (lane == 0) {
                const uint32_t fb = smem_u32(&sh.full[slot]);
                mbar_expect_tx_only(fb, bytes);
                tma_load_2d(s_ring + slot * RS, m, x, y, fb);
                mbar_arrive_n(fb, RING_ARRIVALS);
            }
            __syncwarp();
            return true;
        };
        // two boxes of `bytes` each in one slot (the second at offset `bytes`); nbox = 1 or 2
        auto push_tma2 = [&](const CUtensorMap* m0, int x0, int y0, const CUtensorMap* m1, int x1, int y1,
                             uint32_t bytes, int nbox) -> bool {
            int slot;
            if (!take_slot(slot, false)) return false;
            if (lane == 0) {
                const uint32_t fb = smem_u32(&sh.full[slot]);
                mbar_expect_tx_only(fb, bytes * nbox);
                tma_load_2d(s_ring + slot * RS, m0, x0, y0, fb);
                if (nbox > 1) tma_load_2d(s_ring + slot * RS + bytes, m1, x1, y1, fb);
                mbar_arrive_n(fb, RING_ARRIVALS);
            }
            __syncwarp();
            return true;
        };
        auto push_gather = [&](bool isv, const __nv_bfloat16* src, const int32_t* sel, int h, int j,
                               int nk) -> bool {
            int slot;
            if (!take_slot(slot, SPLIT && isv)) return false;
            const uint32_t dst = s_ring + slot * RS;
            if (!PAIR) {
                // 128 rows x 8 chunks of 16 B: lane l copies chunk l % 8 of rows 4i + l / 8; the
                // 32 row indices are loaded first (independent loads), then the copies are issued
                const int c = lane & 7;
                int rows[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int tok = j * 128 + 4 * i + (lane >> 3);
                    rows[i] = tok < nk ? __ldg(sel + tok) : -1;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = 4 * i + (lane >> 3);
                    const bool okr = rows[i] >= 0;
                    cp_async16(swz(dst, r, c), src + ((size_t)h * N + (okr ? rows[i] : 0)) * 64 + c * 8, okr);
                }
            } else if (!isv) {
                // keys: this CTA's 64 tokens of the block, 8 chunks each (128 B swizzle)
                const int c = lane & 7;
                int rows[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int tok = j * 128 + 64 * (int)crank + 4 * i + (lane >> 3);
                    rows[i] = tok < nk ? __ldg(sel + tok) : -1;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = 4 * i + (lane >> 3);
                    const bool okr = rows[i] >= 0;
                    cp_async16(swz(dst, r, c), src + ((size_t)h * N + (okr ? rows[i] : 0)) * 64 + c * 8, okr);
                }
            } else {
                // values: all 128 tokens, this CTA's 32 head dimensions = 4 chunks (64 B swizzle)
                const int c = lane & 3;
                int rows[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int tok = j * 128 + 8 * i + (lane >> 2);
                    rows[i] = tok < nk ? __ldg(sel + tok) : -1;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = 8 * i + (lane >> 2);
                    const bool okr = rows[i] >= 0;
                    cp_async16(swz64(dst, r, c),
                               src + ((size_t)h * N + (okr ? rows[i] : 0)) * 64 + 32 * crank + c * 8, okr);
                }
            }
            // each lane arrives once its own copies landed: the warp never waits for them
            cp_async_mbar_arrive_noinc(smem_u32(&sh.full[slot]));
            return true;
        };
        const int rb = (int)crank * BR;   // this CTA's row offset inside a 128-row B tile
        for (int64_t it = it0; it < n_iter && ok; it += it_step) {
            if (!active(it)) continue;
            const Unit u = unit_at(it, crank);
            const int nk = u.sel ? a.ksel : N;
            const int nb = (nk + 127) / 128;
            auto push_kv = [&](bool isv, int h, int j) -> bool {
                if (u.sel) return push_gather(isv, isv ? Vg : Kg, u.sel, h, j, nk);
                if (isv) return push_tma(&tm_v, PAIR ? 32 * (int)crank : 0, h * N + j * 128, PAIR ? 8192 : SLOT, SPLIT);
                return push_tma(&tm_k, 0, h * N + j * 128 + rb, BR * 128);
            };
            if constexpr (SPLIT) {
                // blocks b = h nb + j of all heads in one stream: the Q projection of every head first
                // (C/128 items of Wq rows), keys three blocks ahead of their values
                const int nbt = H * nb;
                if (!vprod) {
                    for (int i = 0; i < C / 128 && ok; ++i) ok = push_tma(&tm_wq, 0, i * 128, 128 * 128);
                    for (int b = 0; b < nbt && b < NSB && ok; ++b) ok = push_kv(false, b / nb, b % nb);
                }
                for (int b = 0; b < nbt && ok; ++b) {
                    if (vprod) ok = push_kv(true, b / nb, b % nb);
                    else if (b + NSB < nbt) ok = push_kv(false, (b + NSB) / nb, (b + NSB) % nb);
                }
            } else {
                for (int h = 0; h < H && ok; ++h) {
                    ok = push_tma(&tm_wq64, 0, h * 64 + (PAIR ? 32 * (int)crank : 0), PAIR ? 32 * 128 : 64 * 128);
                    for (int j = 0; j < nb && j < NSB && ok; ++j) ok = push_kv(false, h, j);
                    for (int j = 0; j < nb && ok; ++j) {
                        ok = push_kv(true, h, j);
                        if (j + NSB < nb) ok = ok && push_kv(false, h, j + NSB);
                    }
                }
            }
            if (vprod) continue;   // the value producer has no weight items
            // X = PE Wq^T + a Wo^T : items of AT K atoms (atom 0: Wq, atom ka > 0: Wo columns ka-1)
            for (int nc = 0; nc < C / 128 && ok; ++nc)
                for (int ka = 0; ka < KA && ok; ka += AT) {
                    const CUtensorMap* m0 = ka == 0 ? &tm_wq : &tm_wo;
                    const int x0 = ka == 0 ? 0 : (ka - 1) * 64;
                    ok = push_tma2(m0, x0, nc * 128 + rb, &tm_wo, ka * 64, nc * 128 + rb, BR * 128,
                                   ka + AT <= KA ? AT : KA - ka);
                }
            // MLP items in MMA consumption order
            for (int hf = 0; hf < n_half && ok; ++hf) {
                auto w1 = [&](int c) {
                    for (int s = 0; s < w1_gran && ok; s += AT)
                        ok = push_tma2(&tm_w1, s * 64, c * HN + rb, &tm_w1, (s + 1) * 64, c * HN + rb, BR * 128, AT);
                };
                auto w2 = [&](int c) {
                    for (int q = 0; q < w2_gran && ok; q += AT) {
                        const int nc = q / (HN / 64), kh = q % (HN / 64);
                        ok = push_tma2(&tm_w2, c * HN + kh * 64, hf * 256 + nc * 128 + rb, &tm_w2,
                                       c * HN + (kh + 1) * 64, hf * 256 + nc * 128 + rb, BR * 128, AT);
                    }
                };
                w1(0);
                if (n_chunks > 1) w1(1);
                for (int c = 0; c < n_chunks && ok; ++c) {
                    w2(c);
                    if (c + 2 < n_chunks) w1(c + 2);
                }
            }
        }
        // every load issued has landed before the CTA may exit (they always
        // complete; consumed or not, the last use of each slot is awaited;
        // in the even CTA of a pair that includes the odd CTA's forwarded half)
        if (lane == 0) {
            const uint32_t first = head_a > (uint32_t)NRA ? head_a - NRA : 0;
            for (uint32_t i = first; i < head_a; ++i) drain_wait(smem_u32(&sh.full[i % NRA]), (i / NRA) & 1, ta.timeout);
            if constexpr (NRB > 0) {
                const uint32_t fb = head_b > (uint32_t)NRB ? head_b - NRB : 0;
                for (uint32_t i = fb; i < head_b; ++i)
                    drain_wait(smem_u32(&sh.full[NRA + i % NRB]), (i / NRB) & 1, ta.timeout);
            }
        }
        __syncwarp();
    }
    // ==================================================================== MMA issue
    else if (warp == WARP_MMA && PAIR && !leader) {
        // odd CTA of a pair: forward the completion of each of its ring loads to the
        // even CTA's ring barrier, item by item in ring order
        {
            int f_slot = 0;
            uint32_t f_ph = 0;
            bool ok = true;
            for (int64_t it = it0; it < n_iter && ok; it += it_step) {
                if (!active(it)) continue;
                const Unit u = unit_at(it, crank);
                const int nb = ((u.sel ? a.ksel : N) + 127) / 128;
                const int items = n_items(nb);
                for (int i = 0; i < items && ok; ++i) {
                    uint32_t ph = f_ph;
                    if (!(ok = W.wait(&sh.full[f_slot], ph, 49))) break;
                    fence_proxy_async();   // gathered rows (cp.async) become visible to the async proxy
                    // the phase has completed (the half tile is in place), so the arrival itself orders nothing
                    mbar_arrive_cluster_relaxed_w(mapa(smem_u32(&sh.full[f_slot]), 0u));
                    if (++f_slot == NR) {
                        f_slot = 0;
                        f_ph ^= 1;
                    }
                }
            }
        }
    }
    else if (warp == WARP_MMA) {
        {   // the whole warp runs the issue loop; one elected lane issues each instruction
            // the MMA issuer of a pair waits on barriers that the other CTA arrives at
            W.cluster_acq = PAIR;
            uint32_t ph_pe = 0, ph_qc = 0, ph_p[2] = {0, 0}, ph_a = 0, ph_hin = 0, ph_r = 0, ph_g[2] = {0, 0};
            uint32_t ph_hd = 0, ph_w2 = 0, ph_pvm = 0 /* bit k: phase of bar_pvm[k] (bit 0 alone: pairs) */;
            int ev_pvm = 0;   // P V completions awaited so far (single CTAs)
            bool ok = true;
            int c_slot = 0;
            uint32_t c_ph = 0;
            auto consume = [&](int& slot) -> bool {
                slot = c_slot;
                uint32_t ph = c_ph;
                if (!W.wait(&sh.full[slot], ph, 50)) return false;
                tc_fence_after();
                if (++c_slot == NRA) {
                    c_slot = 0;
                    c_ph ^= 1;
                }
                return true;
            };
            auto release = [&](int slot) { commit_both(&sh.empty[slot]); };
            constexpr int MR = 128 * CG;   // MMA rows
            auto mma_s = [&](uint32_t d, uint64_t da, uint64_t db, uint32_t id, uint32_t acc) {
                if (PAIR) mma_ss_pair_w(d, da, db, id, acc);
                else mma_ss_w(d, da, db, id, acc);
            };
            auto mma_t = [&](uint32_t d, uint32_t ta_, uint64_t db, uint32_t id, uint32_t acc) {
                if (PAIR) mma_ts_pair_w(d, ta_, db, id, acc);
                else mma_ts_w(d, ta_, db, id, acc);
            };
            int64_t n_done = 0;
            for (int64_t it = it0; it < n_iter && ok; it += it_step) {
                if (!active(it)) continue;
                const Unit u = unit_at(it, crank);
                const bool first_unit = n_done++ == 0;
                const int nk = u.sel ? a.ksel : N;
                const int nb = (nk + 127) / 128;
                if (!(ok = W.wait(&sh.bar_pe, ph_pe, 51))) break;
                tc_fence_after();
                if constexpr (SPLIT) {
                    // Q of every head first: PE Wq^T in C/128 items of 128 output rows, into TMEM [0, C)
                    for (int i = 0; i < C / 128 && ok; ++i) {
                        int slot;
                        if (!(ok = consume(slot))) break;
                        const uint64_t da = desc_sw128(s_pe), db = desc_sw128(s_ring + slot * RS);
                        #pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_s(tmem + 128 * i, da + 2 * kk, db + 2 * kk, idesc_bf16(MR, 128, false), kk > 0);
                        release(slot);
                    }
                    if (!ok) break;
                    if (!(ta.inject && first_unit)) commit_both(&sh.bar_q);
                    // every head's packed Q is in shared memory (and the accumulators are read)
                    if (!(ok = W.wait(&sh.bar_qc, ph_qc, 52))) break;
                    tc_fence_after();
                    // then the blocks b = h nb + j of all heads as one stream: S_b into buffer b mod 3,
                    // signalled on bar_s[(b mod 3) * 2 + j mod 2] (one waiting warpgroup per barrier);
                    // S_{b+3} waits for P V_b, which reads P_b from the same columns
                    const int nbt = H * nb;
                    auto issue_sb = [&](int b) -> bool {
                        const int h = b / nb, j = b - h * nb;
                        int sl;
                        if (!consume(sl)) return false;
                        // gathered rows were written by cp.async (generic proxy): order them before the MMA's reads
                        if (u.sel) fence_proxy_async();
                        const uint64_t da = desc_sw128(s_abuf + h * 16384), db = desc_sw128(s_ring + sl * RS);
                        const uint32_t sd = tmem + T_S0 + 128 * (b % NSB);
                        #pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_s(sd, da + 2 * kk, db + 2 * kk, idesc_bf16(MR, 128, false), kk > 0);
                        release(sl);
                        commit_both(&sh.bar_s[(b % NSB) * 2 + (j & 1)]);
                        return true;
                    };
                    for (int b = 0; b < nbt && b < NSB && ok; ++b) ok = issue_sb(b);
                    for (int b = 0; b + NSB < nbt && ok; ++b) {
                        const int e = ev_pvm % 3;
                        uint32_t ph = (ph_pvm >> e) & 1u;
                        if (!(ok = W.wait(&sh.bar_pvm[e], ph, 66))) break;
                        ph_pvm ^= 1u << e;
                        ++ev_pvm;
                        tc_fence_after();
                        ok = issue_sb(b + NSB);
                    }
                    if (!ok) break;
                } else
                for (int h = 0; h < H && ok; ++h) {
                    int slot;
                    // Q_h = PE Wq_h^T (M=128, N=64, K=64)
                    if (!(ok = consume(slot))) break;
                    {
                        const uint64_t da = desc_sw128(s_pe), db = desc_sw128(s_ring + slot * RS);
                        #pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_s(tmem + T_QACC, da + 2 * kk, db + 2 * kk, idesc_bf16(MR, 64, false), kk > 0);
                        release(slot);
                        if (!(ta.inject && h == 0 && first_unit)) commit_both(&sh.bar_q);
                    }
                    if (!(ok = W.wait(&sh.bar_qc, ph_qc, 52))) break;
                    tc_fence_after();
                    auto issue_s = [&](int j) -> bool {
                        int sl;
                        if (!consume(sl)) return false;
                        // gathered rows were written by cp.async (generic proxy): order them before the MMA's reads
                        if (u.sel) fence_proxy_async();
                        const uint64_t da = desc_sw128(s_abuf + h * 16384), db = desc_sw128(s_ring + sl * RS);
                        const uint32_t sd = tmem + T_S0 + 128 * (j % NSB);
                        #pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_s(sd, da + 2 * kk, db + 2 * kk, idesc_bf16(MR, 128, false), kk > 0);
                        release(sl);
                        commit_both(&sh.bar_s[j % 6]);
                        return true;
                    };
                    for (int j = 0; j < nb && j < NSB && ok; ++j) ok = issue_s(j);
                    {
                    for (int j = 0; j < nb && ok; ++j) {
                        const int g = j & 1;   // block j belongs to warpgroup j mod 2
                        if (!(ok = W.wait(&sh.bar_p[g], ph_p[g], 53))) break;
                        tc_fence_after();
                        if (!(ok = consume(slot))) break;
                        if (u.sel) fence_proxy_async();
                        // O_g += P_j V_j. P_j is read in place: the bf16 pairs of tokens [32i, 32i+32)
                        // occupy columns [32i, 32i+16) of its S buffer. V is N-major: 16 tokens per
                        // k-step = 16 rows of 128 B (64 B per CTA of a pair)
                        const uint64_t dv = PAIR ? desc_sw64(s_ring + slot * RS) : desc_sw128(s_ring + slot * RS);
                        constexpr int vstep = PAIR ? 64 : 128;
                        const uint32_t pa = tmem + T_S0 + 128 * (j % NSB);
                        #pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_t(tmem + (g ? T_O1 : T_O0), pa + 32 * (kk >> 1) + 8 * (kk & 1), dv + vstep * kk,
                                  idesc_bf16(MR, 64, true), (j >= 2 || kk > 0));
                        release(slot);
                        // O_g is final for this block once the PV is done (the owner waits before its next)
                        if (j + 2 < nb) commit_both(&sh.bar_pvg[g]);
                        if (j + NSB < nb) {
                            // S_{j+3} overwrites the columns this PV reads: let the PV finish first
                            commit_own(&sh.bar_pvm[0]);
                            if (!(ok = W.wait(&sh.bar_pvm[0], ph_pvm, 66))) break;
                            tc_fence_after();
                            ok = issue_s(j + NSB);
                        }
                    }
                    if (!ok) break;
                    commit_both(&sh.bar_pv);   // the head's PVs are complete: O0 and O1 final
                    // the next head's Q projection accumulates in S2, which this head's PVs read
                    commit_own(&sh.bar_hd);
                    if (!(ok = W.wait(&sh.bar_hd, ph_hd, 54))) break;
                    tc_fence_after();
                    }
                }
                if (!ok) break;
                // ---- X = PE Wq^T + a Wo^T
                if (!(ok = W.wait(&sh.bar_a, ph_a, 55))) break;
                tc_fence_after();
                for (int nc = 0; nc < C / 128 && ok; ++nc)
                    for (int ka0 = 0; ka0 < KA && ok; ka0 += AT) {
                        int slot;
                        if (!(ok = consume(slot))) break;
                        for (int at = 0; at < AT && ka0 + at < KA; ++at) {
                            const int ka = ka0 + at;
                            const uint64_t da = desc_sw128(ka == 0 ? s_pe : s_abuf + (ka - 1) * 16384);
                            const uint64_t db = desc_sw128(s_ring + slot * RS + at * BR * 128);
                            #pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_s(tmem + nc * 128, da + 2 * kk, db + 2 * kk, idesc_bf16(MR, 128, false),
                                      (ka > 0 || kk > 0));
                        }
                        release(slot);
                    }
                if (!ok) break;
                commit_both(&sh.bar_x);
                // ---- MLP
                if (!(ok = W.wait(&sh.bar_hin, ph_hin, 56))) break;
                tc_fence_after();
                for (int hf = 0; hf < n_half && ok; ++hf) {
                    auto issue_w1 = [&](int c) -> bool {
                        const uint32_t hd = tmem + ((c & 1) ? T_H1 : T_H0);
                        for (int ka0 = 0; ka0 < NA; ka0 += AT) {
                            int sl;
                            if (!consume(sl)) return false;
                            #pragma unroll
                            for (int at = 0; at < AT; ++at) {
                                const int ka = ka0 + at;
                                const uint64_t da = desc_sw128(s_abuf + ka * 16384);
                                const uint64_t db = desc_sw128(s_ring + sl * RS + at * BR * 128);
                                #pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    mma_s(hd, da + 2 * kk, db + 2 * kk, idesc_bf16(MR, HN, false), (ka > 0 || kk > 0));
                            }
                            release(sl);
                        }
                        commit_both(&sh.bar_h[c & 1]);
                        return true;
                    };
                    auto issue_w2 = [&](int c) -> bool {
                        const uint32_t ha = tmem + ((c & 1) ? T_H1 : T_H0);
                        for (int q0 = 0; q0 < w2_gran; q0 += AT) {
                            int sl;
                            if (!consume(sl)) return false;
                            #pragma unroll
                            for (int at = 0; at < AT; ++at) {
                                const int q = q0 + at;
                                const int nc = q / (HN / 64), kh = q % (HN / 64);
                                const uint64_t db = desc_sw128(s_ring + sl * RS + at * BR * 128);
                                #pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    mma_t(tmem + nc * 128, ha + split_col(4 * kh + kk, HN), db + 2 * kk,
                                          idesc_bf16(MR, 128, false), 1u);
                            }
                            release(sl);
                        }
                        return true;
                    };
                    ok = issue_w1(0) && (n_chunks < 2 || issue_w1(1));
                    if (ok && hf == 1) {
                        // the first hidden chunks do not touch the accumulator; W2 needs the restored x1
                        if (!(ok = W.wait(&sh.bar_r, ph_r, 57))) break;
                        tc_fence_after();
                    }
                    for (int c = 0; c < n_chunks && ok; ++c) {
                        if (!(ok = W.wait(&sh.bar_g[c & 1], ph_g[c & 1], 58))) break;
                        tc_fence_after();
                        if (!(ok = issue_w2(c))) break;
                        if (c + 2 < n_chunks) {
                            // H[c%2] is re-written by W1(c+2): W2(c) must have read it first
                            commit_own(&sh.bar_w2);
                            if (!(ok = W.wait(&sh.bar_w2, ph_w2, 59))) break;
                            tc_fence_after();
                            ok = issue_w1(c + 2);
                        }
                    }
                    if (!ok) break;
                    commit_both(&sh.bar_acc);   // the half's accumulator is complete
                }
            }
            // nothing of ours may run on the tensor cores once TMEM is released
            commit_own(&sh.bar_fin);
            drain_wait(smem_u32(&sh.bar_fin), 0, ta.timeout);
        }
    }
    // ==================================================================== P V issue (single CTAs)
    else if (SPLIT && warp == WARP_PV) {
      if constexpr (SPLIT) {
        // O_g += P_j V_j for every block: P_j from its warpgroup, V_j from the value ring
        uint32_t ph_p[2] = {0, 0}, ph_cmb = 0;
        int v_slot = 0;
        uint32_t v_ph = 0;
        int ev = 0;   // completions the S issue waits for (bar_pvm[ev mod 3])
        bool ok = true;
        for (int64_t it = it0; it < n_iter && ok; it += it_step) {
            if (!active(it)) continue;
            const Unit u = unit_at(it, crank);
            const int nk = u.sel ? a.ksel : N;
            const int nb = (nk + 127) / 128;
            const int nbt = H * nb;
            for (int h = 0; h < H && ok; ++h) {
                if (h > 0) {
                    // the first two P V of a head overwrite O0 and O1: the previous head's combine has read them
                    if (!(ok = W.wait(&sh.bar_cmb, ph_cmb, 56))) break;
                    tc_fence_after();
                }
                for (int j = 0; j < nb && ok; ++j) {
                    const int g = j & 1;   // block j belongs to warpgroup j mod 2
                    if (!(ok = W.wait(&sh.bar_p[g], ph_p[g], 53))) break;
                    tc_fence_after();
                    const int slot = NRA + v_slot;
                    {
                        uint32_t ph = v_ph;
                        if (!(ok = W.wait(&sh.full[slot], ph, 91))) break;
                    }
                    tc_fence_after();
                    if (++v_slot == NRB) {
                        v_slot = 0;
                        v_ph ^= 1;
                    }
                    // gathered rows were written by cp.async (generic proxy): order them before the MMA's reads
                    if (u.sel) fence_proxy_async();
                    // P_j is read in place: the bf16 pairs of tokens [32i, 32i+32) occupy columns
                    // [32i, 32i+16) of its S buffer; V is N-major, 16 tokens (rows of 128 B) per k-step
                    const uint64_t dv = desc_sw128(s_ring + slot * RS);
                    const uint32_t pa = tmem + T_S0 + 128 * ((h * nb + j) % NSB);   // block b = h nb + j of the stream
                    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts_w(tmem + (g ? T_O1 : T_O0), pa + 32 * (kk >> 1) + 8 * (kk & 1), dv + 128 * kk,
                                 idesc_bf16(128, 64, true), (j >= 2 || kk > 0));
                    mma_commit_w(smem_u32(&sh.empty[slot]));
                    // O_g is final for this block once the P V is done (the owner waits before its next)
                    if (j + 2 < nb) mma_commit_w(smem_u32(&sh.bar_pvg[g]));
                    if (h * nb + j + NSB < nbt) {   // S of the block three later in the stream waits for it
                        mma_commit_w(smem_u32(&sh.bar_pvm[ev % 3]));
                        ++ev;
                    }
                }
                if (!ok) break;
                mma_commit_w(smem_u32(&sh.bar_pv));   // the head's P V are complete: O0 and O1 final
            }
        }
        // nothing of ours may run on the tensor cores once TMEM is released
        mma_commit_w(smem_u32(&sh.bar_fin2));
        drain_wait(smem_u32(&sh.bar_fin2), 0, ta.timeout);
      }
    }
    // ==================================================================== compute warps
    else {
        const int wg = tid >> 7;             // warpgroup: column half
        const int row = tid & 127;           // query row = TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        uint32_t ph_q = 0, ph_s = 0 /* bit k: phase of bar_s[k] */, ph_pvg[2] = {0, 0}, ph_pv = 0, ph_x = 0, ph_h[2] = {0, 0}, ph_acc = 0, ph_cs = 0,
                 ph_wg = 0;
        const float qscale = 0.125f * kLog2e;
        // smem scratch for row statistics after the attention (the embedding tile is free then)
        float* xs = reinterpret_cast<float*>(dyn_raw + (s_pe - smem_u32(dyn_raw)));
        bool ok = true;
        auto arrive = [&](uint64_t* b) { mbar_arrive(smem_u32(b)); };
        // compute -> MMA signal: per thread, or (CTA pairs) per warp to the even CTA's barrier;
        // every thread has fenced its own stores before it
        auto arrive_mma = [&](uint64_t* b) {
            if (PAIR) {
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(lead_bar(b));
            } else {
                mbar_arrive(smem_u32(b));
            }
        };
        auto wg_sync = [&](int site) -> bool {
            arrive(&sh.bar_wg);
            return W.wait(&sh.bar_wg, ph_wg, site);
        };
        const int HALF = HN / 2;             // hidden units per warpgroup
        float4* park = halves ? reinterpret_cast<float4*>(ta.park) + (size_t)blockIdx.x * (256 / 4) * BM : nullptr;
        for (int64_t it = it0; it < n_iter && ok; it += it_step) {
            if (!active(it)) continue;
            const Unit u = unit_at(it, crank);
            const int nk = u.sel ? a.ksel : N;
            const int nb = (nk + 127) / 128;
            // ---- this row's query
            float p[3] = {0.f, 0.f, 0.f};
            int64_t vox = -1, qid = -1;
            if (row < u.nq) {
                const int64_t slot = u.qbeg + row;
                qid = slot;
                if (a.qmode == kQueryXyz) {
                    p[0] = a.xyz[slot * 3];
                    p[1] = a.xyz[slot * 3 + 1];
                    p[2] = a.xyz[slot * 3 + 2];
                } else if (a.qmode == kQueryGrid) {
                    vox = slot;
                    voxel_point(vox, a.R, p);
                } else {
                    const int64_t pos = a.qlist ? (int64_t)a.qlist[slot] : slot;
                    const int e = a.qorder ? a.qorder[pos] : (int)pos;
                    vox = child_index(a.plist[e >> 3], e & 7, a.R);
                    voxel_point(vox, a.R, p);
                }
            }
            #pragma unroll
            for (int c = 4 * wg; c < 4 * wg + 4; ++c) {
                uint32_t w[4];
                #pragma unroll
                for (int v = 0; v < 4; ++v) w[v] = pack_bf16(pe_lane(p, c * 8 + 2 * v), pe_lane(p, c * 8 + 2 * v + 1));
                st_shared_v4(swz(s_pe, row, c), w);
            }
            fence_proxy_async();
            arrive_mma(&sh.bar_pe);
            float* ml_out = nullptr;
            if (a.probe_ml && row < u.nq && wg == 0) {
                if (a.work == kWorkTileDense) ml_out = a.probe_ml + ((size_t)u.t * a.n_probe + u.first + row) * H * 2;
                else if (a.ml_slot) ml_out = a.probe_ml + (size_t)a.ml_slot[u.qbeg + row] * H * 2;
            }
            // ================================================= attention
            if constexpr (SPLIT) {
                // Q of every head at once (TMEM [64 h, 64 h + 64)): + bq, scaled, bf16 into
                // attention-output atom h, which the head's combine overwrites
                if (!(ok = W.wait(&sh.bar_q, ph_q, 60))) break;
                tc_fence_after();
                for (int h = 0; h < H; ++h) {
                    float q[32], b[32];
                    tmem_ld32(trow + 64 * h + 32 * wg, q);
                    ldg32(a.bq + h * 64 + 32 * wg, b);
                    tmem_wait_ld();
                    reg_fence(q);
                    const uint32_t qa = s_abuf + h * 16384;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t w[4];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int d = 8 * c + 2 * v;
                            w[v] = pack_bf16((q[d] + b[d]) * qscale, (q[d + 1] + b[d + 1]) * qscale);
                        }
                        st_shared_v4(swz(qa, row, 4 * wg + c), w);
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                arrive_mma(&sh.bar_qc);
            }
            for (int h = 0; h < H && ok; ++h) {
              if constexpr (!SPLIT) {
                if (!(ok = W.wait(&sh.bar_q, ph_q, 60))) break;
                tc_fence_after();
                {
                    // dims [32 wg, 32 wg + 32): + bq, scale, bf16 into attention-output atom h (128 B
                    // swizzle), which the head's combine overwrites once its MMAs are done
                    float q[32], b[32];
                    tmem_ld32(trow + T_QACC + 32 * wg, q);
                    ldg32(a.bq + h * 64 + 32 * wg, b);
                    tmem_wait_ld();
                    reg_fence(q);
                    const uint32_t qa = s_abuf + h * 16384;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t w[4];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int d = 8 * c + 2 * v;
                            w[v] = pack_bf16((q[d] + b[d]) * qscale, (q[d + 1] + b[d + 1]) * qscale);
                        }
                        st_shared_v4(swz(qa, row, 4 * wg + c), w);
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                arrive_mma(&sh.bar_qc);
              }
                float m_ref = -INFINITY, l_part = 0.f;
                for (int j = wg; j < nb; j += 2) {
                    // single CTAs: block b = h nb + j of the stream, in buffer b mod 3
                    const int bstr = SPLIT ? h * nb + j : j;
                    {
                        const int sb = SPLIT ? (bstr % NSB) * 2 + (j & 1) : j % 6;
                        uint32_t ph = (ph_s >> sb) & 1u;
                        if (!(ok = W.wait(&sh.bar_s[sb], ph, 61))) break;
                        ph_s ^= 1u << sb;
                    }
                    tc_fence_after();
                    const uint32_t sbase = trow + T_S0 + 128 * (bstr % NSB);
                    const bool first = j < 2;
                    const int valid = nk - j * 128;   // columns < valid are real tokens
                    // block maximum, 64 columns at a time
                    float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
                    #pragma unroll 1
                    for (int c0 = 0; c0 < 128; c0 += 64) {
                        float sa[32], sb[32];
                        tmem_ld32(sbase + c0, sa);
                        tmem_ld32(sbase + c0 + 32, sb);
                        tmem_wait_ld();
                        reg_fence(sa);
                        reg_fence(sb);
                        if (valid < c0 + 64) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) {
                                if (c0 + c >= valid) sa[c] = -INFINITY;
                                if (c0 + 32 + c >= valid) sb[c] = -INFINITY;
                            }
                        }
#pragma unroll
                        for (int c = 0; c < 32; c += 4) {
                            m0 = fmax3(m0, sa[c], sa[c + 1]);
                            m1 = fmax3(m1, sa[c + 2], sa[c + 3]);
                            m2 = fmax3(m2, sb[c], sb[c + 1]);
                            m3 = fmax3(m3, sb[c + 2], sb[c + 3]);
                        }
                    }
                    const float mb = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
                    const bool need = first || (mb > m_ref + 8.0f);
                    const float m_new = need ? fmaxf(mb, m_ref) : m_ref;
                    const float f = (first || m_new == -INFINITY) ? 0.f : ex2(m_ref - m_new);
                    if (need) m_ref = m_new;
                    const float m_use = m_ref == -INFINITY ? 0.f : m_ref;   // no real token yet: P = 0
                    // exponentials, 32 columns at a time; P of columns [c0, c0+32) goes to columns
                    // [c0, c0+16), which are read already
                    // (even and odd columns summed separately, as fp32 pairs)
                    uint64_t lab = f32x2(0.f, 0.f);
                    const uint64_t mm = f32x2(m_use, m_use);
                    #pragma unroll 1
                    for (int c0 = 0; c0 < 128; c0 += 32) {
                        float x[32];
                        tmem_ld32(sbase + c0, x);
                        tmem_wait_ld();
                        reg_fence(x);
                        if (valid < c0 + 32) {
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (c0 + c >= valid) x[c] = -INFINITY;
                        }
                        uint32_t pk[16];
                        if (valid >= c0 + 32) {
                            // the column pairs in kEmuPairs on the FMA pipe, the rest on ex2
#pragma unroll
                            for (int v = 0; v < 16; ++v) {
                                const uint64_t d = sub_f32x2(f32x2(x[2 * v], x[2 * v + 1]), mm);
                                uint64_t e;
                                if ((kEmuPairs >> v) & 1u) {
                                    e = exp2_pair_poly(d);
                                } else {
                                    float d0, d1;
                                    f32x2_split(d, d0, d1);
                                    e = f32x2(ex2(d0), ex2(d1));
                                }
                                lab = add_f32x2(lab, e);
                                float e0, e1;
                                f32x2_split(e, e0, e1);
                                pk[v] = pack_bf16(e0, e1);
                            }
                        } else {
#pragma unroll
                            for (int v = 0; v < 16; ++v) {
                                float d0, d1;
                                f32x2_split(sub_f32x2(f32x2(x[2 * v], x[2 * v + 1]), mm), d0, d1);
                                const float e0 = ex2(d0), e1 = ex2(d1);
                                lab = add_f32x2(lab, f32x2(e0, e1));
                                pk[v] = pack_bf16(e0, e1);
                            }
                        }
                        tmem_st16(sbase + c0, pk);
                    }
                    float la, lb;
                    f32x2_split(lab, la, lb);
                    if (need && !first) l_part *= f;
                    l_part += la + lb;
                    if (!first) {   // the PV of this warpgroup's previous block is done: O_g is stable
                        if (!(ok = W.wait(&sh.bar_pvg[wg], ph_pvg[wg], 62))) break;
                        tc_fence_after();
                    }
                    if (!first && __any_sync(0xffffffffu, need)) {
                        const uint32_t ob = trow + (wg ? T_O1 : T_O0);
                        const float g = need ? f : 1.0f;
                        #pragma unroll 1
                        for (int hh = 0; hh < 4; ++hh) {
                            float o[16];
                            tmem_ld16(ob + 16 * hh, o);
                            tmem_wait_ld();
                            reg_fence16(o);
                            uint32_t uo[16];
#pragma unroll
                            for (int c = 0; c < 16; ++c) uo[c] = __float_as_uint(o[c] * g);
                            tmem_st16(ob + 16 * hh, uo);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    arrive_mma(&sh.bar_p[wg]);
                }
                if (!ok) break;
                if (!(ok = W.wait(&sh.bar_pv, ph_pv, 63))) break;   // PV_{nb-1}
                tc_fence_after();
                // combine the halves: exchange (maximum, sum), then
                // O = (O0 2^(m0-M) + O1 2^(m1-M)) / (l0 2^(m0-M) + l1 2^(m1-M)).
                // CTA pairs exchange through S0, idle until the next head's S_0. Single CTAs stream
                // the next head's scores into the S buffers already, so each thread first reads its
                // first 16 dims of O0 and O1 and then exchanges through the first two of those
                // columns of its own warpgroup's O (which the other warpgroup does not read).
                float o0a[16], o1a[16];
                uint32_t x_own, x_oth;
                if constexpr (SPLIT) {
                    tmem_ld16(trow + T_O0 + 32 * wg, o0a);
                    tmem_ld16(trow + T_O1 + 32 * wg, o1a);
                    tmem_wait_ld();
                    reg_fence16(o0a);
                    reg_fence16(o1a);
                    x_own = trow + (wg ? T_O1 : T_O0) + 32 * wg;
                    x_oth = trow + (wg ? T_O0 : T_O1) + 32 * (wg ^ 1);
                } else {
                    x_own = trow + T_S0 + 2 * wg;
                    x_oth = trow + T_S0 + 2 * (wg ^ 1);
                }
                tmem_st1(x_own, __float_as_uint(m_ref));
                tmem_st1(x_own + 1, __float_as_uint(l_part));
                tmem_wait_st();
                tc_fence_before();
                if (!(ok = wg_sync(70))) break;
                tc_fence_after();
                uint32_t mo_bits = tmem_ld1(x_oth);
                uint32_t lo_bits = tmem_ld1(x_oth + 1);
                tmem_wait_ld();
                asm volatile("" : "+r"(mo_bits), "+r"(lo_bits));
                const float m_oth = __uint_as_float(mo_bits), l_oth = __uint_as_float(lo_bits);
                const bool has_o1 = nb > 1;   // with one block, warpgroup 1 owned none: O1 is unwritten
                const float M = fmaxf(m_ref, m_oth);
                const float f_own = m_ref == -INFINITY ? 0.f : ex2(m_ref - M);
                const float f_oth = m_oth == -INFINITY ? 0.f : ex2(m_oth - M);
                const float l_tot = l_part * f_own + l_oth * f_oth;
                {
                    const float inv = 1.0f / l_tot;
                    const float g0 = (wg ? f_oth : f_own) * inv, g1 = (wg ? f_own : f_oth) * inv;
                    const uint32_t atom = s_abuf + h * 16384;
                    // debug export of the attention output at sampled voxels (fp32, before rounding)
                    float* arow = (a.attn_out && vox >= 0 && vox % a.attn_stride == 0)
                                      ? a.attn_out + (size_t)(vox / a.attn_stride) * C + h * 64 + 32 * wg
                                      : nullptr;
                    #pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {   // 16 of this warpgroup's 32 head dims at a time
                        float o0[16], o1[16];
                        if (SPLIT && hh == 0) {
                            #pragma unroll
                            for (int c = 0; c < 16; ++c) {
                                o0[c] = o0a[c];
                                o1[c] = o1a[c];
                            }
                        } else {
                            tmem_ld16(trow + T_O0 + 32 * wg + 16 * hh, o0);
                            tmem_ld16(trow + T_O1 + 32 * wg + 16 * hh, o1);
                            tmem_wait_ld();
                            reg_fence16(o0);
                            reg_fence16(o1);
                        }
                        #pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            uint32_t w[4];
                            #pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const int d = c * 8 + 2 * v;
                                const float b0 = has_o1 ? o1[d] * g1 : 0.f, b1 = has_o1 ? o1[d + 1] * g1 : 0.f;
                                const float x0 = fmaf(o0[d], g0, b0), x1 = fmaf(o0[d + 1], g0, b1);
                                w[v] = pack_bf16(x0, x1);
                                if (arow) {
                                    arow[16 * hh + d] = x0;
                                    arow[16 * hh + d + 1] = x1;
                                }
                            }
                            st_shared_v4(swz(atom, row, 4 * wg + 2 * hh + c), w);
                        }
                    }
                }
                if (ml_out) {
                    ml_out[h * 2] = M;
                    ml_out[h * 2 + 1] = l_tot;
                }
                if constexpr (SPLIT) {
                    if (h + 1 < H) {   // O0 and O1 are read: the next head's first P V may overwrite them
                        tc_fence_before();
                        arrive(&sh.bar_cmb);
                    }
                }
            }
            if (!ok) break;
            fence_proxy_async();
            tc_fence_before();
            arrive_mma(&sh.bar_a);
            // ================================================= LN1 (each half: C/2 columns)
            if (!(ok = W.wait(&sh.bar_x, ph_x, 64))) break;
            tc_fence_after();
            const int CH = C / 2, c_lo = wg * CH;
            float mean1 = 0.f, rstd1 = 1.f;
            {
                float shift = 0.f, s1 = 0.f, s2 = 0.f;
                for (int cc = c_lo; cc < c_lo + CH; cc += 32) {
                    float v[32], bqv[32], bov[32];
                    tmem_ld32(trow + cc, v);
                    ldg32(a.bq + cc, bqv);
                    ldg32(a.bo + cc, bov);
                    tmem_wait_ld();
                    reg_fence(v);
                    if (cc == c_lo) shift = v[0] + bqv[0] + bov[0];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float d = v[e] + bqv[e] + bov[e] - shift;
                        s1 += d;
                        s2 = fmaf(d, d, s2);
                    }
                }
                const float mh = shift + s1 / (float)CH;
                const float m2h = fmaxf(s2 - s1 * (s1 / (float)CH), 0.f);
                xs[(wg * 128 + row) * 2] = mh;
                xs[(wg * 128 + row) * 2 + 1] = m2h;
                if (!(ok = wg_sync(71))) break;
                const float mo = xs[((wg ^ 1) * 128 + row) * 2], m2o = xs[((wg ^ 1) * 128 + row) * 2 + 1];
                const float m_a = wg ? mo : mh, m_b = wg ? mh : mo;   // fixed order: identical in both halves
                const float d = m_b - m_a;
                mean1 = 0.5f * (m_a + m_b);
                const float m2 = (wg ? m2o : m2h) + (wg ? m2h : m2o) + d * d * 0.25f * (float)C;
                if (a.query_ln) rstd1 = rsqrtf(m2 / (float)C + kLnEps);
                for (int cc = c_lo; cc < c_lo + CH; cc += 16) {
                    float v[16], bqv[16], bov[16], g[16], be[16];
                    tmem_ld16(trow + cc, v);
                    ldg16(a.bq + cc, bqv);
                    ldg16(a.bo + cc, bov);
                    if (a.query_ln) {
                        ldg16(a.ln1_g + cc, g);
                        ldg16(a.ln1_b + cc, be);
                    }
                    tmem_wait_ld();
                    reg_fence16(v);
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float y0 = v[2 * e] + bqv[2 * e] + bov[2 * e];
                        float y1 = v[2 * e + 1] + bqv[2 * e + 1] + bov[2 * e + 1];
                        if (a.query_ln) {
                            y0 = (y0 - mean1) * rstd1 * g[2 * e] + be[2 * e];
                            y1 = (y1 - mean1) * rstd1 * g[2 * e + 1] + be[2 * e + 1];
                        }
                        w[e] = pack_bf16(y0, y1);
                    }
                    const uint32_t atom = s_abuf + (cc / 64) * 16384;
                    const int c0 = (cc % 64) / 8;
                    st_shared_v4(swz(atom, row, c0), &w[0]);
                    st_shared_v4(swz(atom, row, c0 + 1), &w[4]);
                }
                if (halves) {
                    // park x1[:, 256 + 128 wg, +128) (fp32) until the second half: four
                    // consecutive columns per 16-byte word, the 128 rows of a word group adjacent
#pragma unroll 1
                    for (int part = 0; part < 4; ++part) {
                        float v[32];
                        tmem_ld32(trow + 256 + 128 * wg + 32 * part, v);
                        tmem_wait_ld();
                        reg_fence(v);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            park[(32 * wg + 8 * part + q) * BM + row] =
                                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            arrive_mma(&sh.bar_hin);
            // ================================================= MLP
            float hs_mean0 = 0.f, hs_m20 = 0.f, hs_dot0 = 0.f, hs_mean1 = 0.f, hs_m21 = 0.f, hs_dot1 = 0.f;
            float hs_dt0 = 0.f, hs_dt1 = 0.f;   // tSDF head dot products
            for (int hf = 0; hf < n_half && ok; ++hf) {
                if (hf == 1) {
                    // restore the parked x1[:, 256 + 128 wg, +128) into the accumulator [128 wg, +128)
#pragma unroll 1
                    for (int part = 0; part < 4; ++part) {
                        uint32_t w[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 t = park[(32 * wg + 8 * part + q) * BM + row];
                            w[4 * q] = __float_as_uint(t.x);
                            w[4 * q + 1] = __float_as_uint(t.y);
                            w[4 * q + 2] = __float_as_uint(t.z);
                            w[4 * q + 3] = __float_as_uint(t.w);
                        }
                        tmem_st32(trow + 128 * wg + 32 * part, w);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    arrive_mma(&sh.bar_r);
                }
                for (int c = 0; c < n_chunks; ++c) {
                    if (!(ok = W.wait(&sh.bar_h[c & 1], ph_h[c & 1], 65))) break;
                    tc_fence_after();
                    const uint32_t hb = trow + ((c & 1) ? T_H1 : T_H0) + HALF * wg;
                    const int f0 = c * HN + HALF * wg;
                    for (int part = 0; part < HALF / 32; ++part) {
                        float v[32], bb[32];
                        tmem_ld32(hb + 32 * part, v);
                        ldg32(a.b1 + f0 + 32 * part, bb);
                        tmem_wait_ld();
                        reg_fence(v);
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e] = gelu_as_pack(v[2 * e] + bb[2 * e], v[2 * e + 1] + bb[2 * e + 1]);
                        tmem_st16(hb + 16 * part, w);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    arrive_mma(&sh.bar_g[c & 1]);
                }
                if (!ok) break;
                if (!(ok = W.wait(&sh.bar_acc, ph_acc, 67))) break;
                tc_fence_after();
                // x2 = acc + bq + bo + b2 on this warpgroup's half of the half's columns
                const int CWH = CW / 2, cb = hf * 256 + wg * CWH;
                float shift = 0.f, s1 = 0.f, s2 = 0.f, dot = 0.f, dot_t = 0.f;
                for (int cc = 0; cc < CWH; cc += 16) {
                    const int col0 = cb + cc;
                    float v[16], bqv[16], bov[16], wv[16];
                    tmem_ld16(trow + wg * CWH + cc, v);
                    ldg16(a.bq + col0, bqv);
                    ldg16(a.bo + col0, bov);
                    ldg16(a.w_head + col0, wv);
                    tmem_wait_ld();
                    reg_fence16(v);
#pragma unroll
                    for (int e = 0; e < 16; ++e) bqv[e] += bov[e];
                    ldg16(a.b2 + col0, bov);
                    if (a.query_ln) {
                        float gv[16];
                        ldg16(a.ln2_g + col0, gv);
#pragma unroll
                        for (int e = 0; e < 16; ++e) wv[e] *= gv[e];
                    }
                    if (cc == 0) shift = v[0] + bqv[0] + bov[0];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float x = v[e] + bqv[e] + bov[e];
                        const float d = x - shift;
                        s1 += d;
                        s2 = fmaf(d, d, s2);
                        dot = fmaf(x, wv[e], dot);
                    }
                    if (a.feat_out && row < u.nq) {   // the block output itself (vecset encoding)
                        float4* fo = reinterpret_cast<float4*>(a.feat_out + (size_t)qid * C + col0);
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            fo[e / 4] = make_float4(v[e] + bqv[e] + bov[e], v[e + 1] + bqv[e + 1] + bov[e + 1],
                                                    v[e + 2] + bqv[e + 2] + bov[e + 2], v[e + 3] + bqv[e + 3] + bov[e + 3]);
                    }
                    if (a.w_tsdf) {   // second head on the same features (weights folded with LN2's gain)
                        float wt[16];
                        ldg16(a.w_tsdf + col0, wt);
                        if (a.query_ln) {
                            float gv[16];
                            ldg16(a.ln2_g + col0, gv);
#pragma unroll
                            for (int e = 0; e < 16; ++e) wt[e] *= gv[e];
                        }
#pragma unroll
                        for (int e = 0; e < 16; ++e) dot_t = fmaf(v[e] + bqv[e] + bov[e], wt[e], dot_t);
                    }
                }
                const float mh = shift + s1 / (float)CWH;
                const float m2h = fmaxf(s2 - s1 * (s1 / (float)CWH), 0.f);
                float* xh = xs + 512 + hf * 1024;
                xh[(wg * 128 + row) * 4] = mh;
                xh[(wg * 128 + row) * 4 + 1] = m2h;
                xh[(wg * 128 + row) * 4 + 2] = dot;
                xh[(wg * 128 + row) * 4 + 3] = dot_t;
                if (!(ok = wg_sync(73))) break;
                const float* ra = xh + row * 4;            // warpgroup 0's values
                const float* rb = xh + (128 + row) * 4;    // warpgroup 1's values
                const float d = rb[0] - ra[0];
                const float mean_h = 0.5f * (ra[0] + rb[0]);
                const float m2_h = ra[1] + rb[1] + d * d * 0.25f * (float)CW;
                const float dot_h = ra[2] + rb[2];
                if (hf == 0) {
                    hs_mean0 = mean_h;
                    hs_m20 = m2_h;
                    hs_dot0 = dot_h;
                    hs_dt0 = ra[3] + rb[3];
                } else {
                    hs_mean1 = mean_h;
                    hs_m21 = m2_h;
                    hs_dot1 = dot_h;
                    hs_dt1 = ra[3] + rb[3];
                }
            }
            if (!ok) break;
            // ================================================= head + output
            if (wg == 0) {
                float dec, traw;
                if (a.query_ln) {
                    float mean, m2;
                    if (n_half == 1) {
                        mean = hs_mean0;
                        m2 = hs_m20;
                    } else {
                        const float d = hs_mean1 - hs_mean0;
                        mean = 0.5f * (hs_mean0 + hs_mean1);
                        m2 = hs_m20 + hs_m21 + d * d * 0.25f * (float)C;
                    }
                    const float rstd = rsqrtf(m2 / (float)C + kLnEps);
                    dec = (hs_dot0 + hs_dot1 - mean * sh.G) * rstd + sh.Bc;
                    traw = (hs_dt0 + hs_dt1 - mean * sh.Gt) * rstd + sh.Bt;
                } else {
                    dec = hs_dot0 + hs_dot1 + sh.Bc;
                    traw = hs_dt0 + hs_dt1 + sh.Bt;
                }
                if (row < u.nq) {
                    float val = dec, sph = 0.f;
                    if (a.spheres) {
                        sph = sphere_union(p, a.spheres, a.n_spheres);
                        val = sph + a.dec_scale * tanhf(dec);
                    }
                    if (a.out) a.out[qid] = val;
                    if (vox >= 0) {
                        if (a.grid) a.grid[vox] = val;
                        if (a.dec_grid) a.dec_grid[vox] = dec;
                        if (a.tsdf_grid) a.tsdf_grid[vox] = tsdf_value(traw, sph, a);
                    }
                }
            }
            // the next tile's first MMA waits for bar_pe, which these threads
            // only arrive at after every TMEM / smem read of this tile (a bounded
            // barrier among the compute threads)
            arrive(&sh.bar_cs);
            if (!(ok = W.wait(&sh.bar_cs, ph_cs, 68))) break;
        }
    }

    // ---------------------------------------------------------------- wind down
    cp_async_commit();   // copies issued without a group, then wait for all of them
    cp_async_wait<0>();
    tc_fence_before();
    __syncthreads();
    // CTA pairs: neither CTA leaves while the other may still reach its shared memory or TMEM
    if (PAIR) cluster_sync();
    tc_fence_after();
    if (warp == 0) {
        if (PAIR) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

__device__ int g_tc_error = 0;

// parking area for the second half of x1 (C == 512): one 128 x 256 fp32 block per CTA
constexpr int kParkCtas = 160;
__device__ float4 g_x1_park[(size_t)kParkCtas * 256 / 4 * BM];

}  // namespace

// 2D bf16 matrix [rows][cols] row-major, box {64 cols, box_rows rows}, 128 B swizzle
vdm_status make_bf16_map(CUtensorMap* m, const void* base, int64_t rows, int cols, int box_rows, int box_cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(VDM_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    // 64-column boxes use 128-byte rows (128 B swizzle), 32-column boxes 64-byte rows (64 B swizzle)
    const CUtensorMapSwizzle sw = box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VDM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return VDM_OK;
}

int* tc_error_word() {
    int* err = nullptr;
    if (cudaGetSymbolAddress((void**)&err, g_tc_error) != cudaSuccess) return nullptr;
    return err;
}

bool tc_supported(const DecodeArgs& a, vdm_dtype dt) {
    if (dt != VDM_BF16) return false;
    if (a.C != 128 && a.C != 256 && a.C != 512) return false;
    if (a.F % 128 != 0) return false;
    return true;
}

size_t tc_smem_bytes(int C, int* ns_out) {
    const size_t fixed = (size_t)(C / 64) * 16384 + 16384 + 1024;
    const int ns = ring_slots(C);
    if (ns_out) *ns_out = ns;
    return fixed + (size_t)ns * SLOT;
}

vdm_status launch_decode_tc(const DecodeArgs& d, cudaStream_t st) {
    int64_t n_units = d.work == kWorkFlat ? (d.M + BM - 1) / BM : (int64_t)d.T * d.slots;
    if (n_units <= 0) return VDM_OK;
    int ns = 0;
    const size_t smem = tc_smem_bytes(d.C, &ns);
    if (ns < 2) return fail(VDM_ERR_INTERNAL, "not enough shared memory for the ring (%d slots)", ns);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms > kParkCtas) sms = kParkCtas;   // one parking block per CTA
    // CTA pairs (256-row MMAs, each CTA loading half of every weight and key tile) when
    // switched on and at least two SMs
    const bool pair = g_debug.single_cta == 0 && sms >= 2;
    const int br = pair ? 64 : 128;   // rows of a 128-row B tile loaded per CTA
    CUtensorMap m_wq, m_wq64, m_wo, m_w1, m_w2, m_k, m_v;
    VDM_TRY(make_bf16_map(&m_wq, d.Wq, d.C, 64, br, 64));
    VDM_TRY(make_bf16_map(&m_wq64, d.Wq, d.C, 64, br / 2, 64));
    VDM_TRY(make_bf16_map(&m_wo, d.Wo, d.C, d.C, br, 64));
    VDM_TRY(make_bf16_map(&m_w1, d.W1, d.F, d.C, br, 64));
    VDM_TRY(make_bf16_map(&m_w2, d.W2, d.C, d.F, br, 64));
    VDM_TRY(make_bf16_map(&m_k, d.K, (int64_t)d.H * d.N, 64, br, 64));
    // values are read N-major: a pair splits the 64 head dimensions, 32 per CTA
    VDM_TRY(make_bf16_map(&m_v, d.V, (int64_t)d.H * d.N, 64, 128, pair ? 32 : 64));
    TcArgs ta;
    ta.d = d;
    ta.ns = ns;
    ta.park = nullptr;
    if (d.C > 256 && cudaGetSymbolAddress((void**)&ta.park, g_x1_park) != cudaSuccess)
        return fail(VDM_ERR_CUDA, "parking area lookup failed");
    ta.err = tc_error_word();
    if (!ta.err) return fail(VDM_ERR_CUDA, "error word lookup failed");
    ta.timeout = g_debug.timeout > 0 ? g_debug.timeout : 4000000000ll;
    // test hook: the g_debug.inject-th launch from the hook's call withholds one signal
    ta.inject = g_debug.inject == 1;
    if (g_debug.inject > 0) --g_debug.inject;
    typedef void (*Kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                         CUtensorMap, TcArgs);
    Kern kern;
    if (pair) kern = d.C == 128 ? decode_tc_kernel<128, 2> : d.C == 256 ? decode_tc_kernel<256, 2> : decode_tc_kernel<512, 2>;
    else kern = d.C == 128 ? decode_tc_kernel<128, 1> : d.C == 256 ? decode_tc_kernel<256, 1> : decode_tc_kernel<512, 1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "decode_tc smem attribute: %s", cudaGetErrorString(e));
    // work items: units of 128 queries, or pairs of them
    const int slots_pairs = pair ? (d.slots + 1) / 2 : d.slots;
    const int64_t n_iter = !pair ? n_units : d.work == kWorkFlat ? (n_units + 1) / 2 : (int64_t)d.T * slots_pairs;
    const int per = pair ? 2 : 1;
    const int64_t groups = sms / per;
    const unsigned grid = (unsigned)(per * (n_iter < groups ? n_iter : groups));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(pair ? NT : NT_SPLIT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = per;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    prof_begin(kProfDecode, st);
    e = cudaLaunchKernelEx(&cfg, kern, m_wq, m_wq64, m_wo, m_w1, m_w2, m_k, m_v, ta);
    prof_end(kProfDecode, st);
    if (e != cudaSuccess) return fail(VDM_ERR_CUDA, "decode_tc_kernel launch: %s", cudaGetErrorString(e));
    return check_launch("decode_tc_kernel");
}

int decode_simt_chunk();

vdm_status launch_decode(DecodeArgs a, vdm_dtype dt, cudaStream_t st) {
    const bool tc = tc_supported(a, dt);
    if (a.work != kWorkFlat) {
        const int qt = tc ? kTcTile : decode_simt_chunk();
        const int most = a.work == kWorkTileDense ? (a.n_probe < 512 ? a.n_probe : 512) : 512 - a.n_probe;
        a.slots = most > 0 ? (most + qt - 1) / qt : 0;
        if (a.slots == 0) return VDM_OK;
    }
    if (tc) return launch_decode_tc(a, st);
    return launch_decode_simt(a, dt, 0, st);
}

// Reads and clears the device error word (call after the stream is synchronised).
vdm_status tc_check_error() {
    int h = 0;
    VDM_CUDA_TRY(cudaMemcpyFromSymbol(&h, g_tc_error, sizeof(int)));
    if (h) {
        int z = 0;
        cudaMemcpyToSymbol(g_tc_error, &z, sizeof(int));
        return fail(VDM_ERR_TIMEOUT, "tensor-core kernel: bounded wait expired at site %d", h);
    }
    return VDM_OK;
}

}  // namespace vdm
