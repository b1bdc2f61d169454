// kv_tc.cuh -- tensor-core dK/dV pass for bf16, d == dv in {64, 128}: the
// key-tile-major half of the backward pass when dQ is computed by its own
// query-tile-major pass (dq_tc.cuh).
//
// A work item is 128 keys (K_j, V_j resident in shared memory) of one (batch,
// head) and the 128-row query tiles i that can see them (i >= j when causal);
// persistent CTAs, one per SM, take the items in order from a counter. Per
// query tile, with keys as the MMA's M dimension:
//   S^T  = K_j Q_i^T                  tcgen05 (A = K_j, B = Q_i, both K-major)
//   dP^T = V_j dO_i^T                 tcgen05 (A = V_j, B = dO_i)
//   P^T  = 2^(S^T*scale*log2e - LSE_i*log2e), 0 where masked        (phase A)
//   dS^T = P^T * (scale*dP^T - scale*D_i)                            (phase B)
//   dV_j += P^T dO_i                  tcgen05, A = P^T from TMEM (bf16 written
//                                     over its own S^T columns), B = dO_i MN-major
//   dK_j += dS^T Q_i                  tcgen05, A = dS^T from TMEM, B = Q_i MN-major
// dV_j and dK_j stay in TMEM across all query tiles and are written once;
// folding `scale` into dS makes dK come out already scaled. With no dQ in
// this pass, nothing here waits on another CTA and no partial sums leave the
// SM.
//
// Two P/dS warpgroups split a tile into four chunks of 32 queries (two chunks
// each) and work on it in two phases. Phase A turns S^T into P^T (it needs
// only S^T); phase B turns dP^T and the P^T kept in registers (bf16, as the
// dV MMA takes it) into dS^T. Each chunk is signalled as soon as its P^T (or
// dS^T) is in TMEM, so the MMA thread issues that chunk's dV (or dK) k-steps
// while the chunks after it are computed; with two warps per SM sub-partition
// each hides the other's latencies. Each chunk's P^T/dS^T go into the first
// 16 of its own 32 TMEM columns, so no chunk overwrites data another chunk has
// yet to read. The MMA thread issues, per tile g: dV(g) chunk by chunk, then
// S^T(g+1) (every MMA that reads P^T(g) is issued by then, and the tensor
// pipe runs MMAs in issue order), then dK(g) chunk by chunk, then dP^T(g+1)
// (likewise after the last reader of dS^T(g)). So the next tile's phase A
// overlaps this tile's dK and dP^T MMAs. Items are ordered in groups of
// heads, key-tile major inside a group (the longest items first when causal),
// so the heads in flight share their Q/dO tiles through L2. An item's dV/dK
// epilogue is staged in the Q/dO stage of its last tile and overlaps the next
// item's first loads.
//
// Where the pages stand: dV, dP, dS and dK are "Attention Backward Pass (dQ,
// dK, dV)", section "Backward", and "Attention backward", Problems 2-6;
// D = rowsum(dO * O) replaces rowsum(dP * P) per "Attention Backpropagation:
// Step by step derivation", section "Gradient of S"; masked dS entries are
// exact zeros ("Attention backward", Problem 8), so tiles wholly above the
// diagonal are skipped.
//
// Warp roles (384 threads): warps 0-3 and 4-7 = the two P/dS warpgroups (TMEM
// lane = key), warp 8 = TMA producer, warp 9 = TMEM allocator and MMA issuer.
// TMEM (512 columns): dV [0,D) dK [D,2D) S^T [2D,2D+128) dP^T [2D+128,2D+256);
// chunk c's P^T (bf16) goes to S^T's columns [32c, 32c+16) and its dS^T to
// dP^T's.
#pragma once

#include "sm100.cuh"
#include "padmask.cuh"

namespace attn {
namespace kvtc {

constexpr int kBN = 128;      // keys per work item
constexpr int kBM = 128;      // queries per tile
constexpr int kChunks = 4;    // 32-query chunks of a tile
constexpr int kThreads = 320;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;

template <int D>
struct Cfg {
    static constexpr int kStages = (D == 64) ? 4 : 2;
    static constexpr int kPanels = D / 64;
    static constexpr int kTileBytes = 128 * D * 2;     // a 128-row bf16 tile
    static constexpr int kPanelBytes = 128 * 128;      // 128 rows x 128 B
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kTileBytes;
    static constexpr int kOffQ = kOffV + kTileBytes;
    static constexpr int kOffdO = kOffQ + kStages * kTileBytes;
    static constexpr int kOffLse = kOffdO + kStages * kTileBytes;
    static constexpr int kOffDd = kOffLse + kStages * kBM * 4;
    static constexpr int kOffBar = kOffDd + kStages * kBM * 4;
    static constexpr int kSmemBytes = kOffBar + 512;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColdV = 0;
    static constexpr uint32_t kColdK = D;
    static constexpr uint32_t kColS = 2 * D;
    static constexpr uint32_t kColdP = 2 * D + 128;
    static constexpr uint32_t kColP = kColS;          // bf16 P^T over S^T
    static constexpr uint32_t kColdS = kColdP;        // bf16 dS^T over dP^T
};
static_assert(Cfg<128>::kSmemBytes <= 232448, "shared memory");

struct Bars {
    uint64_t kv_full;
    uint64_t kv_empty;      // the item's last MMA has read K_j, V_j
    uint64_t q_full[4];
    uint64_t q_empty[4];
    uint64_t s_full;
    uint64_t dp_full;
    uint64_t p_chunk[kChunks];
    uint64_t ds_chunk[kChunks];
    uint64_t acc_done;
    uint64_t acc_free;      // the epilogue has read dV, dK out of TMEM
    uint64_t epi_done[4];   // an item's dV, dK staged in stage s and read by the TMA
    uint64_t mma_drain;
    uint64_t sched_full[4];     // work item of slot k published by the producer
    uint64_t sched_empty[4];    // ... and read by the 9 consumers
    int sched_item[4];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier area");

// Phase A for sixteen queries (columns q0..q0+15 of a tile) of one key row:
// P^T = 2^(S^T * scale * log2(e) - LSE_2) from the S^T values in registers,
// written to TMEM at `pcol` (8 columns, two bf16 per column) and returned
// packed in `pk` for phase B. MASKED applies the causal / key-range mask:
// columns below `keys_masked_below` get P = 0.
template <bool MASKED>
__device__ __forceinline__ void p_half(int q0, const uint32_t (&sr)[16], const float* lse_s,
                                       int keys_masked_below, float scale_log2, uint32_t pcol,
                                       uint32_t* pk) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse_s + q0 + 4 * g);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
        float p[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int e = 4 * g + h;
            p[h] = ex2(fmaf(__uint_as_float(sr[e]), scale_log2, -lv[h]));
            if (MASKED && (q0 + e) < keys_masked_below) p[h] = 0.f;
        }
        pk[2 * g] = pack_bf16x2(p[0], p[1]);
        pk[2 * g + 1] = pack_bf16x2(p[2], p[3]);
    }
    tmem_st8(pcol, pk);
}

// Phase B for the same sixteen queries: dS^T = P^T * (scale * dP^T - scale * D)
// from the dP^T values in registers and phase A's packed P^T (masked entries
// are exact zeros there, so dS^T is too), written to TMEM at `dscol` and
// returned packed in `dk` for the shared-memory tile.
__device__ __forceinline__ void ds_half(int q0, const uint32_t (&pr)[16], const uint32_t* pk,
                                        const float* dd_s, float scale, uint32_t dscol,
                                        uint32_t* dk) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float4 d4 = *reinterpret_cast<const float4*>(dd_s + q0 + 4 * g);
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
        const float p[4] = {__uint_as_float(pk[2 * g] << 16), __uint_as_float(pk[2 * g] & 0xffff0000u),
                            __uint_as_float(pk[2 * g + 1] << 16),
                            __uint_as_float(pk[2 * g + 1] & 0xffff0000u)};
        float ds[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) ds[h] = p[h] * fmaf(__uint_as_float(pr[4 * g + h]), scale, -dv[h]);
        dk[2 * g] = pack_bf16x2(ds[0], ds[1]);
        dk[2 * g + 1] = pack_bf16x2(ds[2], ds[3]);
    }
    tmem_st8(dscol, dk);
}

// The (head, key tile) of work item `b` in schedule order (see the kernel's
// comment).
__device__ __forceinline__ void cta_tile(int b, int num_kt, int BH, int hg, int& bh, int& kt) {
    const int group = b / (hg * num_kt);
    const int within = b % (hg * num_kt);
    const int heads_here = min(hg, BH - group * hg);
    kt = within / heads_here;
    bh = group * hg + within % heads_here;
}

// One work item: 128 keys of one head and the query tiles that see them.
// mk: the head's valid keys (the padding mask, or m). An item whose keys are
// all padding visits one query tile, where every P is 0, so that its dK and
// dV rows are still written (as zeros).
struct Item {
    int bh, k0, first_qt, T, mk;
};
__device__ __forceinline__ Item item_at(int b, int num_kt, int num_qt, int BH, int hg, int causal,
                                        const int* key_len, int H, int m) {
    Item it;
    int kt;
    cta_tile(b, num_kt, BH, hg, it.bh, kt);
    it.k0 = kt * kBN;
    it.mk = keys_valid(key_len, it.bh, H, m);
    it.first_qt = causal ? kt : 0;
    it.T = (it.k0 >= it.mk) ? 1 : num_qt - it.first_qt;          // >= 1
    return it;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
          const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
          const float* __restrict__ lse2, const float* __restrict__ Dd, int* __restrict__ sched,
          int n_pad, int n, int m, int BH, int head_group, int causal, float scale,
          float scale_log2, const int* __restrict__ key_len, int H, unsigned long long budget_ns) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Persistent: G CTAs (at most one per SM). CTA c starts with work item
    // c, and takes every further item from a global counter (zeroed by the
    // preprocess kernel) as it goes, so items are handed out in order to
    // whichever CTA is ready. Items are ordered in groups of `head_group`
    // heads (about 256 items a group, so the heads in flight keep their Q/dO
    // tiles in L2); inside a group key-tile major, so the longest items of the
    // group (lowest key tiles, if causal) come first. The producer publishes
    // each item to the other roles through a 4-slot ring in shared memory,
    // one item ahead.
    const int num_kt = (m + kBN - 1) / kBN;
    const int num_qt = (n + kBM - 1) / kBM;
    const int num_items = num_kt * BH;
    const int G = int(gridDim.x);
    auto item = [&](int b) {
        return item_at(b, num_kt, num_qt, BH, head_group, causal, key_len, H, m);
    };
    // Consumers: the work item of the j-th slot (-1 = no more), or -2 if
    // the wait gave up. A warp reads it in every lane, then lane 0 releases
    // the slot; the MMA thread passes warp = false.
    auto next_item = [&](int j, bool warp_wide) -> int {
        const int slot = j & 3;
        const bool got = warp_wide
                             ? mbar_wait_warp(&bars->sched_full[slot], (j >> 2) & 1, abort_flag, budget_ns)
                             : mbar_wait(&bars->sched_full[slot], (j >> 2) & 1, abort_flag, budget_ns);
        if (!got) return -2;
        const int b = *reinterpret_cast<volatile int*>(&bars->sched_item[slot]);
        if (warp_wide) __syncwarp();
        if (!warp_wide || (threadIdx.x & 31) == 0) mbar_arrive(&bars->sched_empty[slot]);
        return b;
    };

    if (threadIdx.x == 0) {
        // The swizzled tiles need a 1024-byte aligned base. A CTA that starts
        // after another one gave up a wait does no work at all.
        const bool misaligned = (smem_addr(smem) & 1023u) != 0;
        if (misaligned) record_device_error(kErrTimeout);
        bars->abort = (misaligned || *reinterpret_cast<volatile unsigned int*>(&g_device_error) != 0) ? 1 : 0;
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->kv_empty, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->dp_full, 1);
        for (int c = 0; c < kChunks; ++c) {
            mbar_init(&bars->p_chunk[c], 128);
            mbar_init(&bars->ds_chunk[c], 128);
        }
        mbar_init(&bars->acc_done, 1);
        mbar_init(&bars->acc_free, 256);
        for (int s = 0; s < 4; ++s) mbar_init(&bars->epi_done[s], 256);
        mbar_init(&bars->mma_drain, 1);
        for (int k = 0; k < 4; ++k) {
            mbar_init(&bars->sched_full[k], 1);
            mbar_init(&bars->sched_empty[k], 1 + 8);
        }
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
        prefetch_tensor_map(&tmdO);
        prefetch_tensor_map(&tmdK);
        prefetch_tensor_map(&tmdV);
        // Q_i, dO_i and the LSE/D slices of one query tile into stage g % S
        // (g counts query tiles over all of this CTA's items). A stage that
        // held an item's last tile also holds that item's dV/dK epilogue
        // staging: it is reloaded once the epilogue is done with it.
        uint32_t last_in = 0;      // bit s: stage s held an item's last tile
        uint32_t epi_parity = 0;   // bit s: parity of the next epi_done[s] phase
        auto load_q = [&](const Item& it, int t, int g) -> bool {
            const int s = g % C::kStages;
            const int q0 = (it.first_qt + t) * kBM;
            if (g >= C::kStages &&
                !mbar_wait(&bars->q_empty[s], (g / C::kStages - 1) & 1, abort_flag, budget_ns))
                return false;
            if ((last_in >> s) & 1u) {
                if (!mbar_wait(&bars->epi_done[s], (epi_parity >> s) & 1u, abort_flag, budget_ns))
                    return false;
                epi_parity ^= 1u << s;
            }
            last_in = (last_in & ~(1u << s)) | (uint32_t(t == it.T - 1) << s);
            mbar_arrive_expect_tx(&bars->q_full[s], 2 * C::kTileBytes + 2 * kBM * 4);
            for (int p = 0; p < C::kPanels; ++p) {
                tma_load_3d(smem + C::kOffQ + s * C::kTileBytes + p * C::kPanelBytes, &tmQ,
                            &bars->q_full[s], p * 64, q0, it.bh);
                tma_load_3d(smem + C::kOffdO + s * C::kTileBytes + p * C::kPanelBytes, &tmdO,
                            &bars->q_full[s], p * 64, q0, it.bh);
            }
            bulk_load(smem + C::kOffLse + s * kBM * 4, lse2 + size_t(it.bh) * n_pad + q0, kBM * 4,
                      &bars->q_full[s]);
            bulk_load(smem + C::kOffDd + s * kBM * 4, Dd + size_t(it.bh) * n_pad + q0, kBM * 4,
                      &bars->q_full[s]);
            return true;
        };
        auto publish = [&](int k, int b) -> bool {
            const int slot = k & 3;
            if (k >= 4 &&
                !mbar_wait(&bars->sched_empty[slot], ((k >> 2) - 1) & 1, abort_flag, budget_ns))
                return false;
            bars->sched_item[slot] = b;
            mbar_arrive(&bars->sched_full[slot]);
            return true;
        };
        int g = 0, kv_issued = 0;
        int b = int(blockIdx.x);
        bool ok = publish(0, b);
        for (int j = 0; ok; ++j) {
            const Item it = item(b);
            // The first query tile goes in as soon as a stage is free; K_j and
            // V_j once the previous item's last MMA has read its own.
            if (!load_q(it, 0, g)) { ok = false; break; }
            ++g;
            if (j > 0 && !mbar_wait(&bars->kv_empty, (j - 1) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p) {
                tma_load_3d(smem + C::kOffK + p * C::kPanelBytes, &tmK, &bars->kv_full, p * 64, it.k0, it.bh);
                tma_load_3d(smem + C::kOffV + p * C::kPanelBytes, &tmV, &bars->kv_full, p * 64, it.k0, it.bh);
            }
            ++kv_issued;
            for (int t = 1; t < it.T; ++t) {
                if (!load_q(it, t, g)) { ok = false; break; }
                ++g;
            }
            if (!ok) break;
            // All of this item's loads are issued (a couple of tiles ahead of
            // the MMAs): take the next item now, publish it, and warm L2 with
            // its K/V.
            int nb = G + atomicAdd(sched, 1);
            if (nb >= num_items) nb = -1;
            if (!publish(j + 1, nb)) { ok = false; break; }
            if (nb < 0) break;
            const Item nx = item(nb);
            for (int p = 0; p < C::kPanels; ++p) {
                tma_prefetch_l2_3d(&tmK, p * 64, nx.k0, nx.bh);
                tma_prefetch_l2_3d(&tmV, p * 64, nx.k0, nx.bh);
            }
            b = nb;
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: every load issued must land before the CTA may exit. Loads
        // older than the last stage's worth (and K/V before the last) were
        // consumed, so they have landed.
        if (kv_issued > 0) (void)mbar_wait_timed(&bars->kv_full, (kv_issued - 1) & 1, budget_ns);
        for (int t = (g > C::kStages ? g - C::kStages : 0); t < g; ++t)
            (void)mbar_wait_timed(&bars->q_full[t % C::kStages], (t / C::kStages) & 1, budget_ns);
    } else if (!aborted_early && warp == kWarpMma) {
        // ------------------------------------------------ MMA issuer
        // The whole warp walks the loop (waits are warp-wide) and one elected
        // lane issues the MMAs and commits.
        const uint32_t leader = elect_leader();
        constexpr uint32_t idSP = idesc_bf16_f32(kBN, kBM, 0, 0);   // S^T, dP^T
        constexpr uint32_t idKV = idesc_bf16_f32(kBN, D, 0, 1);     // dV, dK
        const uint32_t sK = smem_addr(smem + C::kOffK);
        const uint32_t sV = smem_addr(smem + C::kOffV);
        // S^T(g) = K Q(g)^T and dP^T(g) = V dO(g)^T once Q/dO(g) are in;
        // s_full / dp_full report them.
        auto issue_S = [&](int g) -> bool {
            const int s = g % C::kStages;
            if (!mbar_wait_warp(&bars->q_full[s], (g / C::kStages) & 1, abort_flag, budget_ns)) return false;
            tc_fence_after();
            const uint32_t sQ = smem_addr(smem + C::kOffQ + s * C::kTileBytes);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::kColS, sdesc_at(sK, koff, 16, 1024),
                         sdesc_at(sQ, koff, 16, 1024), idSP, kk > 0, leader);
            }
            mma_commit_w(&bars->s_full, leader);
            return true;
        };
        auto issue_dP = [&](int g) {
            const uint32_t sdO = smem_addr(smem + C::kOffdO + (g % C::kStages) * C::kTileBytes);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::kColdP, sdesc_at(sV, koff, 16, 1024),
                         sdesc_at(sdO, koff, 16, 1024), idSP, kk > 0, leader);
            }
            mma_commit_w(&bars->dp_full, leader);
        };
        bool ok = true;
        int g = 0;
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const int T = item(b).T;
            if (!mbar_wait_warp(&bars->kv_full, j & 1, abort_flag, budget_ns) || !issue_S(g)) {
                ok = false;
                break;
            }
            issue_dP(g);
            for (int t = 0; t < T; ++t, ++g) {
                const int s = g % C::kStages;
                const uint32_t sQ = smem_addr(smem + C::kOffQ + s * C::kTileBytes);
                const uint32_t sdO = smem_addr(smem + C::kOffdO + s * C::kTileBytes);
                // The item's first dV MMA overwrites the accumulators: the
                // previous item's epilogue must have read them out.
                if (t == 0 && j > 0 &&
                    !mbar_wait_warp(&bars->acc_free, (j - 1) & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                // dV += P^T dO per chunk as a P/dS warpgroup has written that
                // chunk's P^T (32 queries, two k-steps; the two warpgroups
                // finish chunks 0 and 2 first, then 1 and 3).
                bool first = (t == 0);
                for (int ci = 0; ci < kChunks; ++ci) {
                    const int c = (ci >> 1) | ((ci & 1) << 1);        // 0, 2, 1, 3
                    if (!mbar_wait_warp(&bars->p_chunk[c], g & 1, abort_flag, budget_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int kk = 2 * c + h;                      // queries 16kk..16kk+15
                        mma_ts_w(tmem + C::kColdV, tmem + C::kColP + 32 * c + 8 * h,
                                 sdesc_at(sdO, kk * 2048, C::kPanelBytes, 1024), idKV, !first, leader);
                        first = false;
                    }
                }
                if (!ok) break;
                // S^T(g+1): every MMA that reads P^T(g) has been issued.
                if (t + 1 < T && !issue_S(g + 1)) { ok = false; break; }
                // dK += dS^T Q per chunk as phase B has written its dS^T.
                first = (t == 0);
                for (int ci = 0; ci < kChunks; ++ci) {
                    const int c = (ci >> 1) | ((ci & 1) << 1);
                    if (!mbar_wait_warp(&bars->ds_chunk[c], g & 1, abort_flag, budget_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int kk = 2 * c + h;
                        mma_ts_w(tmem + C::kColdK, tmem + C::kColdS + 32 * c + 8 * h,
                                 sdesc_at(sQ, kk * 2048, C::kPanelBytes, 1024), idKV, !first, leader);
                        first = false;
                    }
                }
                if (!ok) break;
                mma_commit_w(&bars->q_empty[s], leader);
                // dP^T(g+1): every MMA that reads dS^T(g) has been issued.
                if (t + 1 < T) issue_dP(g + 1);
                if (t == T - 1) {
                    mma_commit_w(&bars->acc_done, leader);
                    mma_commit_w(&bars->kv_empty, leader);      // K_j, V_j free once these complete
                }
            }
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        mma_commit_w(&bars->mma_drain, leader);
        (void)mbar_wait_timed(&bars->mma_drain, 0, budget_ns);
    } else if (!aborted_early && warp < 8) {
        // ------------------------------------------------ P / dS warpgroups
        const int grp = warp >> 2;                       // chunks 2*grp and 2*grp+1
        const int r = threadIdx.x & 127;                 // key row in the tile == TMEM lane
        const uint32_t tl = tmem + (uint32_t((warp & 3) * 32) << 16);
        bool ok = true;
        int g = 0;
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const Item it = item(b);
            const bool key_ok = it.k0 + r < it.mk;
            for (int t = 0; t < it.T; ++t, ++g) {
                const int s = g % C::kStages;
                const int q0 = (it.first_qt + t) * kBM;
                if (!mbar_wait_warp(&bars->q_full[s], (g / C::kStages) & 1, abort_flag, budget_ns) ||
                    !mbar_wait_warp(&bars->s_full, g & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float* lse_s = reinterpret_cast<const float*>(smem + C::kOffLse + s * kBM * 4);
                const float* dd_s = reinterpret_cast<const float*>(smem + C::kOffDd + s * kBM * 4);
                // Keys past the end get P = 0 in every column; on the diagonal
                // tile, key r is masked for the queries in the tile before it
                // (q < r). The masked variant is chosen per warp, never per
                // lane: it holds warp-collective tcgen05.st instructions, which
                // must not sit in a divergent branch. Lanes that need no mask
                // get a bound of 0.
                const bool diag = causal && (q0 == it.k0);
                const int below = !key_ok ? kBM : (diag ? r : 0);
                const bool masked = __any_sync(0xffffffffu, below > 0);
                // Both phases walk four half-chunks of 16 queries (two chunks),
                // each half's TMEM load issued while the previous half is
                // computed. A chunk's P^T/dS^T go into the first 16 of its own
                // 32 columns: half h of chunk c writes columns 32c+8h..32c+8h+7,
                // which it has read.
                uint32_t pk0[16], pk1[16], ds0[16], ds1[16];   // ds*: scratch for ds_half
                uint32_t bA[16], bB[16];
                const int cbase = 2 * grp;
                // Phase A: P^T from S^T.
                tmem_ld16(tl + C::kColS + cbase * 32, bA);
                tmem_ld_wait();
#pragma unroll
                for (int hc = 0; hc < 4; ++hc) {
                    const int c = cbase + (hc >> 1), half = hc & 1;
                    const int qcol = 32 * c + 16 * half;              // first query of the half
                    uint32_t (&cur)[16] = (hc & 1) ? bB : bA;
                    uint32_t (&nxt)[16] = (hc & 1) ? bA : bB;
                    if (hc < 3) {
                        const int qn = 32 * (cbase + ((hc + 1) >> 1)) + 16 * ((hc + 1) & 1);
                        tmem_ld16(tl + C::kColS + qn, nxt);
                    }
                    uint32_t* pk = ((hc >> 1) ? pk1 : pk0) + 8 * half;
                    const uint32_t pcol = tl + C::kColP + 32 * c + 8 * half;
                    if (masked)
                        p_half<true>(qcol, cur, lse_s, below, scale_log2, pcol, pk);
                    else
                        p_half<false>(qcol, cur, lse_s, below, scale_log2, pcol, pk);
                    if (half == 1) {
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(&bars->p_chunk[c]);
                    }
                    if (hc < 3) tmem_ld_wait();
                }
                // Phase B: dS^T from dP^T and the packed P^T.
                if (!mbar_wait_warp(&bars->dp_full, g & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_ld16(tl + C::kColdP + cbase * 32, bA);
                tmem_ld_wait();
#pragma unroll
                for (int hc = 0; hc < 4; ++hc) {
                    const int c = cbase + (hc >> 1), half = hc & 1;
                    const int qcol = 32 * c + 16 * half;
                    uint32_t (&cur)[16] = (hc & 1) ? bB : bA;
                    uint32_t (&nxt)[16] = (hc & 1) ? bA : bB;
                    if (hc < 3) {
                        const int qn = 32 * (cbase + ((hc + 1) >> 1)) + 16 * ((hc + 1) & 1);
                        tmem_ld16(tl + C::kColdP + qn, nxt);
                    }
                    const uint32_t* pk = ((hc >> 1) ? pk1 : pk0) + 8 * half;
                    uint32_t* dk = ((hc >> 1) ? ds1 : ds0) + 8 * half;
                    ds_half(qcol, cur, pk, dd_s, scale, tl + C::kColdS + 32 * c + 8 * half, dk);
                    if (half == 1) {
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(&bars->ds_chunk[c]);
                    }
                    if (hc < 3) tmem_ld_wait();
                }
            }
            if (!ok) break;
            // Epilogue of item j: group 0 writes dV, group 1 writes dK, staged
            // in the Q / dO halves of the stage that held the item's last tile
            // (every MMA that read it is complete once acc_done has fired; the
            // producer reloads it only after epi_done). Each thread reads its
            // key row out of TMEM 32 columns at a time, converts it to bf16
            // and stages it in the 128-byte swizzled layout of the output's
            // tensor map; one lane per warp stores 32 x 64 boxes with the TMA
            // (rows past m clipped). The accumulators are released for the
            // next item as soon as they have been read.
            if (!mbar_wait_warp(&bars->acc_done, j & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                const int s_last = (g - 1) % C::kStages;
                const uint32_t col = grp == 0 ? C::kColdV : C::kColdK;
                uint8_t* stage = smem + (grp == 0 ? C::kOffQ : C::kOffdO) + s_last * C::kTileBytes +
                                 (warp & 3) * (32 * D * 2);
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t rr[32];
                    tmem_ld32(tl + col + 32 * q, rr);
                    tmem_ld_wait(rr);
                    uint8_t* buf = stage + (q >> 1) * 4096;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int kc = 4 * (q & 1) + k;            // 16-byte chunk of the 128-byte row
                        *reinterpret_cast<uint4*>(buf + lane * 128 + ((kc ^ (lane & 7)) * 16)) = make_uint4(
                            pack_bf16x2(__uint_as_float(rr[8 * k + 0]), __uint_as_float(rr[8 * k + 1])),
                            pack_bf16x2(__uint_as_float(rr[8 * k + 2]), __uint_as_float(rr[8 * k + 3])),
                            pack_bf16x2(__uint_as_float(rr[8 * k + 4]), __uint_as_float(rr[8 * k + 5])),
                            pack_bf16x2(__uint_as_float(rr[8 * k + 6]), __uint_as_float(rr[8 * k + 7])));
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->acc_free);
                const CUtensorMap* out_map = grp == 0 ? &tmdV : &tmdK;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int pnl = 0; pnl < C::kPanels; ++pnl)
                        tma_store_3d(out_map, stage + pnl * 4096, 64 * pnl, it.k0 + 32 * (warp & 3), it.bh);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
                __syncwarp();
                mbar_arrive(&bars->epi_done[s_last]);
            }
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

}  // namespace kvtc
}  // namespace attn
