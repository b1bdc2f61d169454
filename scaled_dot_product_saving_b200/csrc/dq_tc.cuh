// dq_tc.cuh -- tensor-core dQ pass for bf16, d == dv in {64, 128}: the
// query-tile-major half of the backward pass (the other half, dK and dV, is
// kv_tc.cuh). Each query tile's dQ is summed over its key tiles inside one
// CTA and written once, in bf16: no accumulator in global memory, no atomics
// and no conversion pass.
//
// A work item is one 128-row query tile i of one (batch, head), with Q_i and
// dO_i resident in shared memory, walking the key tiles j that it sees (j <= i
// when causal, and only tiles with a valid key under the padding mask). Per
// key tile, with queries as the MMA's M dimension:
//   S  = Q_i K_j^T                    tcgen05 (A = Q_i, B = K_j, both K-major)
//   dP = dO_i V_j^T                   tcgen05 (A = dO_i, B = V_j)
//   P  = 2^(S*scale*log2e - LSE_i*log2e), 0 where masked            (phase A)
//   dS = P * (scale*dP - scale*D_i)                                  (phase B)
//   dQ_i += dS K_j                    tcgen05, A = dS from TMEM (bf16 written
//                                     over its own S columns), B = K_j MN-major
// The scale is folded into dS, so dQ comes out scaled. P is rebuilt from the
// forward's LSE and kept in registers (bf16, as in the dK/dV pass) between
// the two phases; D is the preprocess kernel's rowsum(dO * O).
//
// Where the pages stand: dQ = scale * dS K is "Attention backward", Problem
// 5, and "Attention Backward Pass (dQ, dK, dV)", section "Backward"; dS is
// Problem 4 there, with D = rowsum(dO * O) from "Attention Backpropagation:
// Step by step derivation", section "Gradient of S"; masked entries of P and
// dS are exact zeros (Problem 8), so key tiles wholly past the diagonal or the
// valid keys are never visited.
//
// Pipeline. S is double-buffered in TMEM, so the MMA thread issues, per key
// tile c (counted over the CTA's whole walk): dP(c) once phase B of tile c-1
// has read dP(c-1), S(c+1) into the other buffer, then dQ += dS(c) K_j once
// phase B of tile c has written dS(c). The tensor pipe runs MMAs in issue
// order, so S(c+1) overwrites dS(c-1) only after the dQ MMA that reads it.
// Phase A of tile c+1 thus overlaps the dQ MMA of tile c and the dP MMA of
// tile c+1.
//
// Warp roles (320 threads): warps 0-3 and 4-7 = two elementwise warpgroups,
// warpgroup h handling keys [64h, 64h+64) of every query row (warp w reads
// TMEM lanes 32(w%4) .. 32(w%4)+31, one query row per thread); warp 8 = TMA
// producer; warp 9 = TMEM allocator and MMA issuer.
// TMEM (512 columns): S buffers [0,128) and [128,256), dP [256,384), dQ
// [384, 384+D). Keys [64h, 64h+64) of a tile's dS (bf16, two per column) go to
// columns [64h, 64h+32) of its S buffer.
// Shared memory: Q_i, dO_i (each also the staging buffer of nothing: dQ is
// stored straight from registers), then K and V rings.
#pragma once

#include "sm100.cuh"
#include "padmask.cuh"

namespace attn {
namespace dqtc {

constexpr int kBM = 128;      // queries per tile
constexpr int kBN = 128;      // keys per tile
constexpr int kThreads = 320;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;

template <int D>
struct Cfg {
    static constexpr int kKStages = (D == 64) ? 4 : 3;
    static constexpr int kVStages = (D == 64) ? 4 : 2;
    static constexpr int kPanels = D / 64;              // 64-column swizzle panels
    static constexpr int kTileBytes = kBM * D * 2;      // a 128-row bf16 tile
    static constexpr int kPanelBytes = kBM * 128;       // 128 rows x 128 B
    static constexpr int kOffQ = 0;
    static constexpr int kOffdO = kOffQ + kTileBytes;
    static constexpr int kOffK = kOffdO + kTileBytes;
    static constexpr int kOffV = kOffK + kKStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
    static constexpr int kSmemBytes = kOffBar + 512;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0;                // S buffer b at 128 b
    static constexpr uint32_t kColdP = 256;
    static constexpr uint32_t kColdQ = 384;
};
static_assert(Cfg<128>::kSmemBytes <= 232448, "shared memory");

struct Bars {
    uint64_t q_full;            // Q_i, dO_i of the current item in
    uint64_t q_empty;           // the item's last S and dP MMAs have read them
    uint64_t k_full[4];
    uint64_t k_empty[4];
    uint64_t v_full[4];
    uint64_t v_empty[4];
    uint64_t s_full[2];         // S(c) in buffer c % 2
    uint64_t dp_full;           // dP(c)
    uint64_t dp_free;           // phase B has read dP(c)
    uint64_t ds_full;           // phase B has written dS(c)
    uint64_t dq_done;           // the item's last dQ MMA is complete
    uint64_t dq_free;           // the epilogue has read dQ out of TMEM
    uint64_t sched_full[4];     // work item of slot k published by the producer
    uint64_t sched_empty[4];    // ... and read by the MMA thread and the 8 elementwise warps
    uint64_t mma_drain;
    int sched_item[4];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier area");

// Work item `b` -> (head, query tile). Heads go in groups of `hg`; within a
// group the query tiles are taken from the last (most key tiles under the
// causal mask) to the first, each across the group's heads.
struct Item {
    int bh, qt, nkv, mk;
};
__device__ __forceinline__ Item item_at(int b, int num_qt, int BH, int hg, int causal,
                                        const int* key_len, int H, int m) {
    Item it;
    const int group = b / (hg * num_qt);
    const int within = b % (hg * num_qt);
    const int heads_here = min(hg, BH - group * hg);
    it.qt = num_qt - 1 - within / heads_here;
    it.bh = group * hg + within % heads_here;
    it.mk = keys_valid(key_len, it.bh, H, m);
    const int num_kt = (it.mk + kBN - 1) / kBN;           // key tiles with a valid key, >= 1
    it.nkv = causal ? min(num_kt, it.qt + 1) : num_kt;
    return it;
}

// Phase A for one 32-key chunk of a query row: P = 2^(S * scale_log2 -
// lse2), exactly 0 for keys after kmax when MASKED, packed to bf16 pairs.
template <bool MASKED>
__device__ __forceinline__ void chunk_p(const uint32_t (&sr)[32], float scale_log2, float lse2,
                                        int key0, int kmax, uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        float p0 = ex2(fmaf(__uint_as_float(sr[2 * e]), scale_log2, -lse2));
        float p1 = ex2(fmaf(__uint_as_float(sr[2 * e + 1]), scale_log2, -lse2));
        if (MASKED) {
            if (key0 + 2 * e > kmax) p0 = 0.f;
            if (key0 + 2 * e + 1 > kmax) p1 = 0.f;
        }
        pk[e] = pack_bf16x2(p0, p1);
    }
}

// Phase B for one 32-key chunk: dS = P * (scale * dP - dd), with dd = scale *
// D of the row, from phase A's packed P, packed to bf16 pairs.
__device__ __forceinline__ void chunk_ds(const uint32_t (&dpr)[32], const uint32_t* pk,
                                         float scale, float dd, uint32_t (&dsk)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float p0 = __uint_as_float(pk[e] << 16), p1 = __uint_as_float(pk[e] & 0xffff0000u);
        dsk[e] = pack_bf16x2(p0 * fmaf(__uint_as_float(dpr[2 * e]), scale, -dd),
                             p1 * fmaf(__uint_as_float(dpr[2 * e + 1]), scale, -dd));
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
          const float* __restrict__ lse2, const float* __restrict__ Dd, int* __restrict__ sched,
          __nv_bfloat16* __restrict__ dQ, int n_pad, int n, int m, int BH, int head_group,
          int causal, float scale, float scale_log2, const int* __restrict__ key_len, int H,
          unsigned long long budget_ns) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Persistent: G CTAs (at most one per SM). CTA c starts with work item c
    // and takes every further item from a global counter (zeroed by the
    // preprocess kernel), so items go out in order to whichever CTA is ready.
    // The producer publishes each item to the other roles through a 4-slot
    // ring in shared memory, one item ahead.
    const int num_qt = (n + kBM - 1) / kBM;
    const int num_items = num_qt * BH;
    const int G = int(gridDim.x);
    auto item = [&](int b) { return item_at(b, num_qt, BH, head_group, causal, key_len, H, m); };
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
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
            mbar_init(&bars->sched_full[s], 1);
            mbar_init(&bars->sched_empty[s], 1 + 8);
        }
        mbar_init(&bars->s_full[0], 1);
        mbar_init(&bars->s_full[1], 1);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->dp_free, 256);
        mbar_init(&bars->ds_full, 256);
        mbar_init(&bars->dq_done, 1);
        mbar_init(&bars->dq_free, 256);
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
        prefetch_tensor_map(&tmdO);
        auto publish = [&](int k, int b) -> bool {
            const int slot = k & 3;
            if (k >= 4 &&
                !mbar_wait(&bars->sched_empty[slot], ((k >> 2) - 1) & 1, abort_flag, budget_ns))
                return false;
            bars->sched_item[slot] = b;
            mbar_arrive(&bars->sched_full[slot]);
            return true;
        };
        int b = int(blockIdx.x);
        bool ok = publish(0, b);
        int gt = 0, k_issued = 0, v_issued = 0, q_issued = 0;
        for (int j = 0; ok; ++j) {
            const Item it = item(b);
            // Q_i and dO_i, once the previous item's last S and dP MMAs have
            // read their buffers.
            if (j > 0 && !mbar_wait(&bars->q_empty, (j - 1) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            mbar_arrive_expect_tx(&bars->q_full, 2 * C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p) {
                tma_load_3d(smem + C::kOffQ + p * C::kPanelBytes, &tmQ, &bars->q_full, p * 64,
                            it.qt * kBM, it.bh);
                tma_load_3d(smem + C::kOffdO + p * C::kPanelBytes, &tmdO, &bars->q_full, p * 64,
                            it.qt * kBM, it.bh);
            }
            ++q_issued;
            for (int t = 0; t < it.nkv; ++t, ++gt) {
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
            }
            if (!ok) break;
            // All of this item's loads are issued: take the next item.
            int nb = G + atomicAdd(sched, 1);
            if (nb >= num_items) nb = -1;
            if (!publish(j + 1, nb)) { ok = false; break; }
            if (nb < 0) break;
            b = nb;
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: every load issued lands before the CTA may exit. Loads older
        // than a ring's worth were consumed, so they have landed; so were all
        // Q/dO loads before the last.
        if (q_issued > 0) (void)mbar_wait_timed(&bars->q_full, (q_issued - 1) & 1, budget_ns);
        for (int t = (k_issued > C::kKStages ? k_issued - C::kKStages : 0); t < k_issued; ++t)
            (void)mbar_wait_timed(&bars->k_full[t % C::kKStages], (t / C::kKStages) & 1, budget_ns);
        for (int t = (v_issued > C::kVStages ? v_issued - C::kVStages : 0); t < v_issued; ++t)
            (void)mbar_wait_timed(&bars->v_full[t % C::kVStages], (t / C::kVStages) & 1, budget_ns);
    } else if (!aborted_early && warp == kWarpMma) {
        // ------------------------------------------------ MMA issuer
        // The whole warp walks the loop (waits are warp-wide) and one elected
        // lane issues the MMAs and commits.
        const uint32_t leader = elect_leader();
        constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, 0, 0);   // S, dP
        constexpr uint32_t idQ = idesc_bf16_f32(kBM, D, 0, 1);     // dQ (B = K_j MN-major)
        const uint32_t sQ = smem_addr(smem + C::kOffQ);
        const uint32_t sdO = smem_addr(smem + C::kOffdO);
        auto issue_S = [&](int c, int g) {
            const uint32_t sK = smem_addr(smem + C::kOffK + (g % C::kKStages) * C::kTileBytes);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::kColS0 + 128 * (c & 1), sdesc_at(sQ, koff, 16, 1024),
                         sdesc_at(sK, koff, 16, 1024), idS, kk > 0, leader);
            }
            mma_commit_w(&bars->s_full[c & 1], leader);
        };
        auto issue_dP = [&](int g) {
            const uint32_t sV = smem_addr(smem + C::kOffV + (g % C::kVStages) * C::kTileBytes);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::kColdP, sdesc_at(sdO, koff, 16, 1024),
                         sdesc_at(sV, koff, 16, 1024), idS, kk > 0, leader);
            }
            mma_commit_w(&bars->dp_full, leader);
        };
        bool ok = true;
        int gt = 0, c = 0;                     // key tiles so far: in the rings, and overall
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const Item it = item(b);
            if (!mbar_wait_warp(&bars->q_full, j & 1, abort_flag, budget_ns) ||
                !mbar_wait_warp(&bars->k_full[gt % C::kKStages], (gt / C::kKStages) & 1, abort_flag,
                                budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            issue_S(c, gt);
            for (int t = 0; t < it.nkv; ++t, ++c) {
                const int g = gt + t;
                // dP(c), once V_j is in and phase B has read dP(c-1).
                if (!mbar_wait_warp(&bars->v_full[g % C::kVStages], (g / C::kVStages) & 1, abort_flag,
                                    budget_ns) ||
                    (c > 0 && !mbar_wait_warp(&bars->dp_free, (c - 1) & 1, abort_flag, budget_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_dP(g);
                mma_commit_w(&bars->v_empty[g % C::kVStages], leader);
                if (t == it.nkv - 1) mma_commit_w(&bars->q_empty, leader);   // Q_i, dO_i read for the last time
                // S(c+1) into the other buffer, whose dS(c-1) the dQ MMA
                // issued before has read.
                if (t + 1 < it.nkv) {
                    if (!mbar_wait_warp(&bars->k_full[(g + 1) % C::kKStages], ((g + 1) / C::kKStages) & 1,
                                        abort_flag, budget_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_S(c + 1, g + 1);
                }
                // dQ += dS(c) K_j. The item's first one overwrites dQ: the
                // previous item's epilogue must have read it out.
                if ((t == 0 && j > 0 && !mbar_wait_warp(&bars->dq_free, (j - 1) & 1, abort_flag, budget_ns)) ||
                    !mbar_wait_warp(&bars->ds_full, c & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sK = smem_addr(smem + C::kOffK + (g % C::kKStages) * C::kTileBytes);
                const uint32_t sbuf = tmem + C::kColS0 + 128 * (c & 1);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)          // keys 16kk .. 16kk+15
                    mma_ts_w(tmem + C::kColdQ, sbuf + 64 * (kk >> 2) + 8 * (kk & 3),
                             sdesc_at(sK, kk * 2048, C::kPanelBytes, 1024), idQ, t > 0 || kk > 0, leader);
                mma_commit_w(&bars->k_empty[g % C::kKStages], leader);
                if (t == it.nkv - 1) mma_commit_w(&bars->dq_done, leader);
            }
            gt += it.nkv;
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: all MMAs issued here complete before TMEM is released.
        mma_commit_w(&bars->mma_drain, leader);
        (void)mbar_wait_timed(&bars->mma_drain, 0, budget_ns);
    } else if (!aborted_early && warp < 8) {
        // ------------------------------------------------ elementwise warpgroups
        const int h = warp >> 2;                        // keys [64h, 64h + 64) of every row
        const int r = threadIdx.x & 127;                // query row in the tile == TMEM lane
        const uint32_t tl = tmem + (uint32_t((warp & 3) * 32) << 16);
        bool ok = true;
        int c = 0;                                      // key tiles so far, overall
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const Item it = item(b);
            const int row = it.qt * kBM + r;
            // The row's base-2 LSE and scale * D (padded rows: +inf and 0, so
            // their P is 0).
            const float l2 = lse2[size_t(it.bh) * n_pad + row];
            const float dd = Dd[size_t(it.bh) * n_pad + row];
            // Keys after kmax are masked: past the padding mask, or after the
            // row (causal).
            const int kmax = causal ? min(row, it.mk - 1) : it.mk - 1;
            for (int t = 0; t < it.nkv; ++t, ++c) {
                const int key0 = t * kBN + 64 * h;
                const uint32_t ts = tl + C::kColS0 + 128 * (c & 1) + 64 * h;
                // The masked variant is chosen per warp, never per lane: it
                // holds warp-collective tcgen05 instructions.
                const bool masked = __any_sync(0xffffffffu, key0 + 63 > kmax);
                if (!mbar_wait_warp(&bars->s_full[c & 1], (c >> 1) & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // Phase A: P for the 64 keys, kept packed in registers.
                uint32_t pk[32];
                {
                    uint32_t s0[32], s1[32];
                    tmem_ld32(ts, s0);
                    tmem_ld32(ts + 32, s1);
                    tmem_ld_wait(s0);
                    tmem_ld_wait(s1);
                    if (masked) {
                        chunk_p<true>(s0, scale_log2, l2, key0, kmax, pk);
                        chunk_p<true>(s1, scale_log2, l2, key0 + 32, kmax, pk + 16);
                    } else {
                        chunk_p<false>(s0, scale_log2, l2, key0, kmax, pk);
                        chunk_p<false>(s1, scale_log2, l2, key0 + 32, kmax, pk + 16);
                    }
                }
                // Phase B: dS over the S columns already read (chunk q's dS
                // goes to columns 16q .. 16q+15 of this warpgroup's 64).
                if (!mbar_wait_warp(&bars->dp_full, c & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                {
                    uint32_t d0[32], d1[32];
                    tmem_ld32(tl + C::kColdP + 64 * h, d0);
                    tmem_ld32(tl + C::kColdP + 64 * h + 32, d1);
                    tmem_ld_wait(d0);
                    tmem_ld_wait(d1);
                    tc_fence_before();
                    mbar_arrive(&bars->dp_free);
                    uint32_t dsk[16];
                    chunk_ds(d0, pk, scale, dd, dsk);
                    tmem_st16(ts, dsk);
                    chunk_ds(d1, pk + 16, scale, dd, dsk);
                    tmem_st16(ts + 16, dsk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars->ds_full);
            }
            if (!ok) break;
            // Epilogue: dQ of the row's D/2 columns of this warpgroup, to bf16,
            // stored straight from registers (rows past n skipped); dQ is
            // released to the next item's MMAs once read.
            if (!mbar_wait_warp(&bars->dq_done, j & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            __nv_bfloat16* dst = dQ + (size_t(it.bh) * n + row) * D + (D / 2) * h;
#pragma unroll
            for (int q = 0; q < D / 64; ++q) {
                uint32_t v[32];
                tmem_ld32(tl + C::kColdQ + (D / 2) * h + 32 * q, v);
                tmem_ld_wait(v);
                if (q == D / 64 - 1) {
                    tc_fence_before();
                    mbar_arrive(&bars->dq_free);
                }
                if (row < n) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        *reinterpret_cast<uint4*>(dst + 32 * q + 8 * k) = make_uint4(
                            pack_bf16x2(__uint_as_float(v[8 * k + 0]), __uint_as_float(v[8 * k + 1])),
                            pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                            pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                            pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7])));
                }
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

}  // namespace dqtc
}  // namespace attn
