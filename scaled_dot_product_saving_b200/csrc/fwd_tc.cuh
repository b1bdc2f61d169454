// fwd_tc.cuh -- tensor-core forward for bf16, d == dv in {64, 128}.
//
// Computes O = softmax(scale * Q K^T) V and the row log-sum-exp (the forward
// whose softmax statistics the backward recomputes P from: "Attention Backward
// Pass (dQ, dK, dV)", section on the forward; under the causal mask key j > i
// is excluded before the softmax).
//
// A work item is two adjacent 128-row query tiles, A = 2p and B = 2p + 1, of
// one (batch, head), sharing every key and value tile loaded for it; under the
// causal mask B needs one key tile more than A. Items run in groups of heads
// (so a group's keys and values stay in L2), heaviest query rows first within
// a group. The grid has one CTA per item, but the CTAs are persistent: each
// takes over the items of CTAs not yet launched through cluster launch control
// (see the kernel). For each 128-key tile t and each query tile x:
//   S_x = Q_x K_t^T          tcgen05.mma, both operands K-major in shared
//                            memory, fp32 accumulator in TMEM
//   P_x = 2^(S_x * scale * log2e - m_x)   one softmax warpgroup per query
//                            tile, one row (TMEM lane) per thread, m_x the
//                            running row maximum in use
//   O_x += P_x V_t           tcgen05.mma, A = P_x read from TMEM (bf16,
//                            written over the S_x columns it came from),
//                            B = V_t (MN-major), O_x in TMEM
// The MMA thread issues PV_A(t), S_A(t+1), PV_B(t), S_B(t+1), ... so that the
// tensor cores work on one tile while the other tile's softmax runs. The
// softmax hands P over in two halves of 64 keys, and the first half of PV
// starts while the second half of P is computed. Because
// S_x(t+1) is issued after PV_x(t) by the same thread, the barrier that reports
// S_x(t+1) also reports PV_x(t) complete: the softmax may rescale O_x as soon as
// it sees S_x(t+1).
//
// The running maximum is raised, and O rescaled, only when a tile's row
// maximum exceeds the one in use by more than 2^8 in P, so P <= 256 and the
// row sum stays well inside fp32. The exponentials run on the MUFU unit (a
// polynomial on the FMA pipe costs more per element on this part than MUFU.EX2
// does); the scaled scores and the row sums use the paired fp32 instructions,
// which halve their issue slots. At the end O / sum is stored as bf16 through
// shared memory with the TMA, and the row's natural-log LSE as fp32.
//
// Warp roles (320 threads): warps 0-3 softmax of tile A, warps 4-7 softmax of
// tile B (warp w reads TMEM lanes 32(w%4) .. 32(w%4)+31), warp 8 TMA producer,
// warp 9 TMEM allocator and MMA issuer.
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+d),
// O_B [256+d, 256+2d).
// Shared memory: Q_A, Q_B (each also the staging buffer of its O epilogue),
// then K and V rings with their own barriers (a K tile is released as soon as
// both S products that read it are done).
#pragma once

#include "sm100.cuh"
#include "padmask.cuh"

namespace attn {
namespace fwdtc {

constexpr int kBM = 128;      // queries per tile
constexpr int kBN = 128;      // keys per tile
constexpr int kThreads = 320;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
    static constexpr int kKStages = (D == 64) ? 4 : 3;
    static constexpr int kVStages = (D == 64) ? 4 : 2;
    static constexpr int kPanels = D / 64;              // 64-column swizzle panels
    static constexpr int kTileBytes = kBM * D * 2;      // a 128-row bf16 tile
    static constexpr int kPanelBytes = kBM * 128;       // 128 rows x 128 B
    static constexpr int kOffQ = 0;                     // Q_A, Q_B
    static constexpr int kOffK = kOffQ + 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kKStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
    static constexpr int kSmemBytes = kOffBar + 512;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0;                // S_x at kColS0 + 128 x
    static constexpr uint32_t kColO0 = 256;              // O_x at kColO0 + D x
    static constexpr int kStageWarpBytes = 32 * D * 2;  // epilogue: 32 rows per warp
};
static_assert(Cfg<128>::kSmemBytes <= 232448, "shared memory");

struct Bars {
    uint4 clc_resp;             // answer of the last cancellation request (16-byte aligned)
    uint64_t q_full[2];         // Q_x of the current item in
    uint64_t q_free[2];         // Q_x buffer free again (epilogue stored O_x out of it)
    uint64_t k_full[4];
    uint64_t k_empty[4];
    uint64_t v_full[4];
    uint64_t v_empty[4];
    uint64_t s_full[2];
    uint64_t p_half[2];         // P of keys 0..63 of the tile written
    uint64_t p_full[2];         // all of P written
    uint64_t o_done[2];         // last product of the item into O_x complete
    uint64_t o_free[2];         // O_x read out of TMEM by the epilogue
    uint64_t clc_bar;
    uint64_t sched_full[4];     // work item of slot k published by the producer
    uint64_t sched_empty[4];    // ... and read by the MMA thread and the 8 softmax warps
    uint64_t mma_drain;
    int sched_item[4];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier area");

// CTA -> (head, pair of query tiles). Heads go in groups of `hg`; within a
// group the pairs are taken from the last (most key tiles under the causal
// mask) to the first, each across the group's heads.
__device__ __forceinline__ void cta_pair(int b, int num_pairs, int BH, int hg, int& bh, int& pair) {
    const int group = b / (hg * num_pairs);
    const int within = b % (hg * num_pairs);
    const int heads_here = min(hg, BH - group * hg);
    pair = num_pairs - 1 - within / heads_here;
    bh = group * hg + within % heads_here;
}

// Maximum (or, for a negative scale, minimum) of a 32-key chunk of raw scores,
// excluding keys after `kmax` when MASKED; two independent chains.
template <bool NEG, bool MASKED>
__device__ __forceinline__ float chunk_extreme(const uint32_t (&r)[32], int key0, int kmax) {
    float acc[2] = {NEG ? INFINITY : -INFINITY, NEG ? INFINITY : -INFINITY};
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float a = __uint_as_float(r[e]), b = __uint_as_float(r[e + 1]);
        if (MASKED) {
            if (key0 + e > kmax) a = NEG ? INFINITY : -INFINITY;
            if (key0 + e + 1 > kmax) b = NEG ? INFINITY : -INFINITY;
        }
        const int j = (e >> 1) & 1;
        acc[j] = NEG ? fmin3(acc[j], a, b) : fmax3(acc[j], a, b);
    }
    return NEG ? fminf(acc[0], acc[1]) : fmaxf(acc[0], acc[1]);
}

// P for a 32-key chunk: 2^(raw * scale_log2 - m) (exactly 0 for masked keys),
// packed to bf16 pairs in `pk`, summed into `sum` (two chains).
template <bool MASKED>
__device__ __forceinline__ void chunk_p(const uint32_t (&r)[32], f32x2 sl2, f32x2 neg_m,
                                        int key0, int kmax, f32x2 (&sum)[2], uint32_t (&pk)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float2 x = split_f32x2(
            fma_x2(make_f32x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), sl2, neg_m));
        float2 p;
        p.x = ex2(x.x);
        p.y = ex2(x.y);
        if (MASKED) {
            if (key0 + 2 * e > kmax) p.x = 0.f;
            if (key0 + 2 * e + 1 > kmax) p.y = 0.f;
        }
        sum[e & 1] = add_x2(sum[e & 1], make_f32x2(p.x, p.y));
        pk[e] = pack_bf16x2(p.x, p.y);
    }
}

// One work item: the query-tile pair `pair` (tiles A = 2 pair, B = 2 pair + 1)
// of one head, and the key tiles each tile needs.
// mk: the head's valid keys (the padding mask, or m); key tiles past it are
// not visited.
struct Item {
    int bh, qt[2], nkv[2], num_kv, mk;
    bool has_b;
};
__device__ __forceinline__ Item item_at(int b, int num_qt, int BH, int hg, int causal,
                                        const int* key_len, int H, int m) {
    Item it;
    const int num_pairs = (num_qt + 1) / 2;
    int pair;
    cta_pair(b, num_pairs, BH, hg, it.bh, pair);
    it.mk = keys_valid(key_len, it.bh, H, m);
    const int num_kt = (it.mk + kBN - 1) / kBN;
    it.has_b = 2 * pair + 1 < num_qt;
    it.qt[0] = 2 * pair;
    it.qt[1] = 2 * pair + 1;
    it.nkv[0] = causal ? min(num_kt, it.qt[0] + 1) : num_kt;
    it.nkv[1] = it.has_b ? (causal ? min(num_kt, it.qt[1] + 1) : num_kt) : 0;
    it.num_kv = max(it.nkv[0], it.nkv[1]);
    return it;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
           float* __restrict__ LSE, int n, int m, int BH, int head_group, int causal,
           float scale_log2, const int* __restrict__ key_len, int H,
           unsigned long long budget_ns) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_qt = (n + kBM - 1) / kBM;
    auto item = [&](int b) { return item_at(b, num_qt, BH, head_group, causal, key_len, H, m); };
    // Persistent through cluster launch control: a CTA starts with the work
    // item of its own index and, while it works, asks the hardware to cancel
    // the launch of a CTA that has not started and takes over that CTA's item
    // (the hardware answers in launch order, heaviest items first). The
    // producer publishes each item to the other roles through a 4-slot ring
    // in shared memory; -1 ends the walk. next_item returns -2 if a wait gave
    // up.
    auto next_item = [&](int j, bool warp_wide) -> int {
        const int slot = j & 3;
        const bool got = warp_wide
                             ? mbar_wait_warp(&bars->sched_full[slot], (j >> 2) & 1, abort_flag, budget_ns)
                             : mbar_wait(&bars->sched_full[slot], (j >> 2) & 1, abort_flag, budget_ns);
        if (!got) return -2;
        const int b = *reinterpret_cast<volatile int*>(&bars->sched_item[slot]);
        if (warp_wide) __syncwarp();
        if (!warp_wide || lane == 0) mbar_arrive(&bars->sched_empty[slot]);
        return b;
    };

    if (threadIdx.x == 0) {
        // The swizzled tiles need a 1024-byte aligned base. A CTA that starts
        // after another one gave up a wait does no work at all.
        const bool misaligned = (smem_addr(smem) & 1023u) != 0;
        if (misaligned) record_device_error(kErrTimeout);
        bars->abort = (misaligned || *reinterpret_cast<volatile unsigned int*>(&g_device_error) != 0) ? 1 : 0;
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
            mbar_init(&bars->sched_full[s], 1);
            mbar_init(&bars->sched_empty[s], 1 + 8);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->q_full[x], 1);
            mbar_init(&bars->q_free[x], 128);
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->p_half[x], 128);
            mbar_init(&bars->p_full[x], 128);
            mbar_init(&bars->o_done[x], 1);
            mbar_init(&bars->o_free[x], 128);
        }
        mbar_init(&bars->clc_bar, 1);
        mbar_init(&bars->mma_drain, 1);
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&bars->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const bool aborted_early = bars->abort != 0;

    if (!aborted_early && warp == kWarpProducer && lane == 0) {
        // ------------------------------------------------ TMA producer
        prefetch_tensor_map(&tmQ);
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        prefetch_tensor_map(&tmO);
        auto publish = [&](int k, int b) -> bool {
            const int slot = k & 3;
            if (k >= 4 &&
                !mbar_wait(&bars->sched_empty[slot], ((k >> 2) - 1) & 1, abort_flag, budget_ns))
                return false;
            bars->sched_item[slot] = b;
            mbar_arrive(&bars->sched_full[slot]);
            return true;
        };
        // Q_x of an item, once the previous item's epilogue has stored its O_x
        // out of the same buffer.
        int q_uses[2] = {0, 0};
        auto load_q = [&](const Item& it, int x) -> bool {
            if (q_uses[x] > 0 &&
                !mbar_wait(&bars->q_free[x], (q_uses[x] - 1) & 1, abort_flag, budget_ns))
                return false;
            ++q_uses[x];
            mbar_arrive_expect_tx(&bars->q_full[x], C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p)
                tma_load_3d(smem + C::kOffQ + x * C::kTileBytes + p * C::kPanelBytes, &tmQ,
                            &bars->q_full[x], p * 64, it.qt[x] * kBM, it.bh);
            return true;
        };
        int b = int(blockIdx.x);
        bool ok = publish(0, b), stealing = true, clc_pending = false;
        uint32_t clc_phase = 0;
        int gt = 0, k_issued = 0, v_issued = 0;
        for (int j = 0; ok; ++j) {
            const Item it = item(b);
            // Q_A, then K/V tile by tile, with Q_B after the first K/V tile
            // (Q_B waits for the previous item's tile-B epilogue, which ends
            // last).
            if (!load_q(it, 0)) { ok = false; break; }
            for (int t = 0; t < it.num_kv; ++t, ++gt) {
                const int sk = gt % C::kKStages, sv = gt % C::kVStages;
                if (gt >= C::kKStages &&
                    !mbar_wait(&bars->k_empty[sk], (gt / C::kKStages - 1) & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars->k_full[sk], C::kTileBytes);
                for (int p = 0; p < C::kPanels; ++p)
                    tma_load_3d(smem + C::kOffK + sk * C::kTileBytes + p * C::kPanelBytes, &tmK,
                                &bars->k_full[sk], p * 64, t * kBN, it.bh);
                ++k_issued;
                if (gt >= C::kVStages &&
                    !mbar_wait(&bars->v_empty[sv], (gt / C::kVStages - 1) & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars->v_full[sv], C::kTileBytes);
                for (int p = 0; p < C::kPanels; ++p)
                    tma_load_3d(smem + C::kOffV + sv * C::kTileBytes + p * C::kPanelBytes, &tmV,
                                &bars->v_full[sv], p * 64, t * kBN, it.bh);
                ++v_issued;
                if (t == 0 && it.has_b && !load_q(it, 1)) { ok = false; break; }
            }
            if (!ok) break;
            // All of this item's loads are issued (a few key tiles ahead of the
            // MMAs): ask for the next item now.
            int nb = -1;
            if (stealing) {
                mbar_arrive_expect_tx(&bars->clc_bar, 16);
                clc_try_cancel(&bars->clc_resp, &bars->clc_bar);
                clc_pending = true;
                if (!mbar_wait(&bars->clc_bar, clc_phase, abort_flag, budget_ns)) { ok = false; break; }
                clc_phase ^= 1u;
                clc_pending = false;
                int x;
                if (clc_query(&bars->clc_resp, &x)) nb = x;
                else stealing = false;
            }
            if (!publish(j + 1, nb)) { ok = false; break; }
            if (nb < 0) break;
            b = nb;
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: an answer still on its way, and every load issued, land before
        // the CTA may exit. Loads older than a ring's worth were consumed, so
        // they have landed; Q loads before the last of each tile likewise.
        if (clc_pending) (void)mbar_wait_timed(&bars->clc_bar, clc_phase, budget_ns);
        for (int x = 0; x < 2; ++x)
            if (q_uses[x] > 0) (void)mbar_wait_timed(&bars->q_full[x], (q_uses[x] - 1) & 1, budget_ns);
        for (int t = (k_issued > C::kKStages ? k_issued - C::kKStages : 0); t < k_issued; ++t)
            (void)mbar_wait_timed(&bars->k_full[t % C::kKStages], (t / C::kKStages) & 1, budget_ns);
        for (int t = (v_issued > C::kVStages ? v_issued - C::kVStages : 0); t < v_issued; ++t)
            (void)mbar_wait_timed(&bars->v_full[t % C::kVStages], (t / C::kVStages) & 1, budget_ns);
    } else if (!aborted_early && warp == kWarpMma) {
        // ------------------------------------------------ MMA issuer
        // The whole warp walks the loop (waits are warp-wide) and one elected
        // lane issues the MMAs and commits.
        const uint32_t leader = elect_leader();
        constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, 0, 0);
        constexpr uint32_t idO = idesc_bf16_f32(kBM, D, 0, 1);
        auto issue_S = [&](int x, int g) {
            const uint32_t sQ = smem_addr(smem + C::kOffQ + x * C::kTileBytes);
            const uint32_t sK = smem_addr(smem + C::kOffK + (g % C::kKStages) * C::kTileBytes);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::kColS0 + 128 * x, sdesc_at(sQ, koff, 16, 1024),
                         sdesc_at(sK, koff, 16, 1024), idS, kk > 0, leader);
            }
            mma_commit_w(&bars->s_full[x], leader);
        };
        // O_x += P_x V over keys 64h .. 64h+63 of the tile (key tile t of the
        // item, global index g)
        auto issue_PV = [&](int x, int t, int g, int h) {
            const uint32_t sV = smem_addr(smem + C::kOffV + (g % C::kVStages) * C::kTileBytes);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int kk = 4 * h + k4;
                mma_ts_w(tmem + C::kColO0 + D * x, tmem + C::kColS0 + 128 * x + kk * 8,
                         sdesc_at(sV, kk * 2048, C::kPanelBytes, 1024), idO, (t > 0 || kk > 0), leader);
            }
        };
        bool ok = true;
        int gt = 0;
        int cx[2] = {0, 0}, ox[2] = {0, 0}, qx[2] = {0, 0};
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const Item it = item(b);
            // S_x(0) for the active tiles once Q_x and the first K tile are in.
            if (!mbar_wait_warp(&bars->q_full[0], qx[0] & 1, abort_flag, budget_ns) ||
                !mbar_wait_warp(&bars->k_full[gt % C::kKStages], (gt / C::kKStages) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            ++qx[0];
            tc_fence_after();
            issue_S(0, gt);
            if (it.has_b) {
                if (!mbar_wait_warp(&bars->q_full[1], qx[1] & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                ++qx[1];
                tc_fence_after();
                issue_S(1, gt);
            }
            mma_commit_w(&bars->k_empty[gt % C::kKStages], leader);
            for (int t = 0; ok && t < it.num_kv; ++t) {
                const int g = gt + t;
                bool v_ready = false, k_ready = false;
                // For each tile: PV of key tile t once its P is written, then
                // the next S (its columns hold P until that PV has read them;
                // MMAs run in issue order).
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (t >= it.nkv[x]) continue;
                    if (!mbar_wait_warp(&bars->p_half[x], cx[x] & 1, abort_flag, budget_ns)) {
                        ok = false;
                        break;
                    }
                    if (!v_ready) {
                        if (!mbar_wait_warp(&bars->v_full[g % C::kVStages], (g / C::kVStages) & 1,
                                            abort_flag, budget_ns)) {
                            ok = false;
                            break;
                        }
                        v_ready = true;
                    }
                    // The item's first product overwrites O_x: the previous
                    // item's epilogue must have read it out.
                    if (t == 0 && ox[x] > 0 &&
                        !mbar_wait_warp(&bars->o_free[x], (ox[x] - 1) & 1, abort_flag, budget_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_PV(x, t, g, 0);
                    if (!mbar_wait_warp(&bars->p_full[x], cx[x] & 1, abort_flag, budget_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_PV(x, t, g, 1);
                    ++cx[x];
                    if (t + 1 < it.nkv[x]) {
                        if (!k_ready) {
                            if (!mbar_wait_warp(&bars->k_full[(g + 1) % C::kKStages], ((g + 1) / C::kKStages) & 1,
                                                abort_flag, budget_ns)) {
                                ok = false;
                                break;
                            }
                            k_ready = true;
                            tc_fence_after();
                        }
                        issue_S(x, g + 1);
                    } else {
                        mma_commit_w(&bars->o_done[x], leader);   // last product into O_x
                        ++ox[x];
                    }
                }
                if (!ok) break;
                if (k_ready) mma_commit_w(&bars->k_empty[(g + 1) % C::kKStages], leader);
                mma_commit_w(&bars->v_empty[g % C::kVStages], leader);
            }
            gt += it.num_kv;
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: all MMAs issued here complete before TMEM is released.
        mma_commit_w(&bars->mma_drain, leader);
        (void)mbar_wait_timed(&bars->mma_drain, 0, budget_ns);
    } else if (!aborted_early && warp < 8) {
        // ------------------------------------------------ softmax warpgroups
        const int x = warp >> 2;                         // query tile A or B
        const int r = threadIdx.x & 127;                 // row in the tile == TMEM lane
        const uint32_t tl = tmem + (uint32_t((warp & 3) * 32) << 16);
        const uint32_t tS = tl + C::kColS0 + 128 * x, tO = tl + C::kColO0 + D * x;
        const bool neg = scale_log2 < 0.f;
        const f32x2 sl2 = make_f32x2(scale_log2, scale_log2);
        bool ok = true;
        int cx = 0, ox = 0;                              // this tile's key tiles and items so far
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const Item it = item(b);
            if (x == 1 && !it.has_b) continue;
            const int q0 = (x ? it.qt[1] : it.qt[0]) * kBM;
            const int row = q0 + r;
            const int ntile = x ? it.nkv[1] : it.nkv[0];
            // Keys after kmax are masked: past the end or the padding mask,
            // or after the row (causal).
            const int kmax = causal ? min(row, it.mk - 1) : it.mk - 1;
            float m_run = -INFINITY, l_run = 0.f;
            for (int t = 0; t < ntile; ++t) {
                if (!mbar_wait_warp(&bars->s_full[x], cx & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int k0 = t * kBN;
                const bool masked = __any_sync(0xffffffffu, k0 + kBN - 1 > kmax);
                // pass 1: extreme raw score of the row over this key tile
                float ext;
                {
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    tmem_ld32(tS, r0);
                    tmem_ld32(tS + 32, r1);
                    tmem_ld32(tS + 64, r2);
                    tmem_ld32(tS + 96, r3);
                    tmem_ld_wait(r0);
                    tmem_ld_wait(r1);
                    tmem_ld_wait(r2);
                    tmem_ld_wait(r3);
                    float e[4];
                    if (neg) {
                        if (masked) {
                            e[0] = chunk_extreme<true, true>(r0, k0, kmax);
                            e[1] = chunk_extreme<true, true>(r1, k0 + 32, kmax);
                            e[2] = chunk_extreme<true, true>(r2, k0 + 64, kmax);
                            e[3] = chunk_extreme<true, true>(r3, k0 + 96, kmax);
                        } else {
                            e[0] = chunk_extreme<true, false>(r0, k0, kmax);
                            e[1] = chunk_extreme<true, false>(r1, k0 + 32, kmax);
                            e[2] = chunk_extreme<true, false>(r2, k0 + 64, kmax);
                            e[3] = chunk_extreme<true, false>(r3, k0 + 96, kmax);
                        }
                        ext = fminf(fminf(e[0], e[1]), fminf(e[2], e[3]));
                    } else {
                        if (masked) {
                            e[0] = chunk_extreme<false, true>(r0, k0, kmax);
                            e[1] = chunk_extreme<false, true>(r1, k0 + 32, kmax);
                            e[2] = chunk_extreme<false, true>(r2, k0 + 64, kmax);
                            e[3] = chunk_extreme<false, true>(r3, k0 + 96, kmax);
                        } else {
                            e[0] = chunk_extreme<false, false>(r0, k0, kmax);
                            e[1] = chunk_extreme<false, false>(r1, k0 + 32, kmax);
                            e[2] = chunk_extreme<false, false>(r2, k0 + 64, kmax);
                            e[3] = chunk_extreme<false, false>(r3, k0 + 96, kmax);
                        }
                        ext = fmaxf(fmaxf(e[0], e[1]), fmaxf(e[2], e[3]));
                    }
                }
                const float m_new = fmaxf(m_run, ext * scale_log2);
                const bool want = m_new > m_run + kRescaleThreshold;   // true on the first tile
                const bool warp_rescale = __any_sync(0xffffffffu, want && t > 0);
                float alpha = 1.f;
                if (want) {
                    alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
                    m_run = m_new;
                    l_run *= alpha;
                }
                if (warp_rescale) {
                    // O_x holds P(t-1) V(t-1): S_x(t) was issued after that product.
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t rr[32];
                        tmem_ld32(tO + c * 32, rr);
                        tmem_ld_wait(rr);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
                        tmem_st32(tO + c * 32, rr);
                    }
                }
                // pass 2: P as bf16 over the S columns already read (chunk c's P
                // goes to columns 16c .. 16c+15, all read by then)
                const f32x2 neg_m = make_f32x2(-m_run, -m_run);
                f32x2 sum[2] = {make_f32x2(0.f, 0.f), make_f32x2(0.f, 0.f)};
                uint32_t ra[32], rb[32];
                tmem_ld32(tS, ra);
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) {
                    uint32_t(&cur)[32] = (c & 1) ? rb : ra;
                    uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
                    tmem_ld_wait(cur);
                    if (c + 1 < kBN / 32) tmem_ld32(tS + 32 * (c + 1), nxt);
                    uint32_t pk[16];
                    if (masked)
                        chunk_p<true>(cur, sl2, neg_m, k0 + 32 * c, kmax, sum, pk);
                    else
                        chunk_p<false>(cur, sl2, neg_m, k0 + 32 * c, kmax, sum, pk);
                    tmem_st16(tS + 16 * c, pk);
                    if (c == 1) {
                        // keys 0..63 of P are in place: the first half of PV may start
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(&bars->p_half[x]);
                    }
                }
                const float2 s2 = split_f32x2(add_x2(sum[0], sum[1]));
                l_run += s2.x + s2.y;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars->p_full[x]);
                ++cx;
            }
            if (!ok) break;
            if (!mbar_wait_warp(&bars->o_done[x], ox & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            ++ox;
            // Epilogue: O / sum as bf16, staged per warp (32 rows) in the
            // 128B-swizzled layout of O's tensor map inside this tile's Q buffer
            // (no MMA reads it any more), stored with the TMA; rows past n are
            // clipped by the tensor map. LSE in natural log. O_x is released to
            // the next item's MMAs once read, the Q buffer to the producer once
            // the TMA has read it.
            tc_fence_after();
            const float inv = 1.f / l_run;
            uint8_t* stage = smem + C::kOffQ + x * C::kTileBytes + (warp & 3) * C::kStageWarpBytes;
#pragma unroll
            for (int pnl = 0; pnl < C::kPanels; ++pnl) {
                uint32_t ra[32], rb[32];
                tmem_ld32(tO + 64 * pnl, ra);
                tmem_ld32(tO + 64 * pnl + 32, rb);
                tmem_ld_wait(ra);
                tmem_ld_wait(rb);
                uint8_t* buf = stage + pnl * 4096;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t* src = (k < 4) ? ra + 8 * k : rb + 8 * (k - 4);
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(src[0]) * inv, __uint_as_float(src[1]) * inv);
                    w.y = pack_bf16x2(__uint_as_float(src[2]) * inv, __uint_as_float(src[3]) * inv);
                    w.z = pack_bf16x2(__uint_as_float(src[4]) * inv, __uint_as_float(src[5]) * inv);
                    w.w = pack_bf16x2(__uint_as_float(src[6]) * inv, __uint_as_float(src[7]) * inv);
                    *reinterpret_cast<uint4*>(buf + lane * 128 + ((k ^ (lane & 7)) * 16)) = w;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&tmO, buf, 64 * pnl, q0 + 32 * (warp & 3), it.bh);
                    bulk_commit_group();
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->o_free[x]);
            if (row < n) LSE[size_t(it.bh) * n + row] = (m_run + log2f(l_run)) * kLn2;
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            mbar_arrive(&bars->q_free[x]);
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fwdtc
}  // namespace attn
