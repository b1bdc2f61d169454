// bwd_tc.cuh -- tensor-core backward for bf16, d == dv in {64, 128}.
//
// Key-tile major. A work item is 128 keys (K_j, V_j resident in shared memory)
// of one (batch, head) and the 128-row query tiles i that can see them (i >= j
// when causal); persistent CTAs, one per SM, take the items in order from a
// counter (see the kernel). Per query tile, with keys as the MMA's M dimension:
//   S^T  = K_j Q_i^T                  tcgen05 (A = K_j, B = Q_i, both K-major)
//   dP^T = V_j dO_i^T                 tcgen05 (A = V_j, B = dO_i)
//   P^T  = 2^(S^T*scale*log2e - LSE_i*log2e), 0 where masked
//   dS^T = P^T * (scale*dP^T - scale*D_i)        (128 threads, one key each)
//   dV_j += P^T dO_i                  tcgen05, A = P^T from TMEM (bf16 written
//                                     over its own S^T columns), B = dO_i MN-major
//   dK_j += dS^T Q_i                  tcgen05, A = dS^T from TMEM, B = Q_i MN-major
//   dQ_i += dS K_j                    tcgen05, A = dS from shared memory
//                                     (MN-major), B = K_j (MN-major); a second
//                                     warpgroup stages the fp32 result in shared
//                                     memory (d = 128: the by then free dS tile)
//                                     and hands it to the TMA engine as tiled
//                                     reduce-adds into the global dQ accumulator.
// dV_j and dK_j stay in TMEM across all query tiles and are written once.
// Folding `scale` into dS makes dK and dQ come out already scaled.
//
// dQ in bf16. Every key tile of a head adds a partial into the head's rows of
// the fp32 accumulator (zeroed by the preprocess kernel). Once the partials of
// a work item have landed, each warp of the dQ warpgroup counts the item in a
// per-head counter in the workspace (a release add; nobody waits on it). Two
// converter warps per CTA take 32-row slabs of dQ in head order from a global
// claim counter, wait (polling with backoff) until every work item of the
// slab's head has been counted, convert the slab's finished sums to bf16 dQ,
// and drop the dead fp32 lines from L2 without writing them back. They run
// beside the pipeline, so heads that finish early are converted while later
// heads are still being computed; every other warp of a CTA joins them once
// its own work has run out, so the last heads, which finish together, are
// converted by all warps of all CTAs. No separate conversion pass runs.
//
// Two P/dS warpgroups split a tile into four chunks of 32 queries (two chunks
// each) and signal each chunk as soon as its P^T/dS^T are in TMEM, so the MMA
// thread issues that chunk's dV/dK k-steps (d = 64: a half's two chunks at a
// time) while the chunks after it are computed; with two warps per SM sub-partition each hides the other's
// latencies. Each chunk's P^T/dS^T go into the first 16 of its own 32 TMEM
// columns, so no chunk overwrites data another chunk has yet to read. dS for
// the dQ MMA is kept in registers and written to shared memory only at the
// end of the tile, by when the dQ warpgroup has normally finished staging the
// previous tile's dQ through that buffer. Items are ordered in groups of
// heads, key-tile major inside a group (the longest items first when causal),
// so the heads in flight share their Q/dO tiles and their slices of the dQ
// accumulator through L2. An item's dV/dK epilogue is the dQ
// warpgroup's: staged in the Q/dO stage of the item's last tile, it overlaps
// the next item's first loads and P/dS work.
//
// Where the pages stand: dV, dP, dS, dQ and dK are "Attention Backward Pass
// (dQ, dK, dV)", section "Backward", and "Attention backward", Problems 2-6;
// D = rowsum(dO * O) replaces rowsum(dP * P) per "Attention Backpropagation:
// Step by step derivation", section "Gradient of S"; masked dS entries are
// exact zeros ("Attention backward", Problem 8), so tiles wholly above the
// diagonal are skipped.
//
// Warp roles (512 threads): warps 0-3 and 4-7 = the two P/dS warpgroups (TMEM
// lane = key), warps 8-11 = dQ warpgroup (TMEM lane = query row), warp 12 =
// TMA producer, warp 13 = TMEM allocator and MMA issuer (the whole warp walks
// the issue loop, one elected lane issues), warps 14-15 = dQ converters.
//
// TMEM (512 columns). d = 128: dV [0,128) dK [128,256) S^T [256,384)
// dP^T [384,512); chunk c's P^T (bf16) goes to [256+32c, 256+32c+16) and its
// dS^T to [384+32c, 384+32c+16); dQ then takes all of [256,384). The tensor
// pipe runs MMAs in issue order, so the dQ MMA, issued after the last dV MMA,
// overwrites P^T only once it has been read; the next tile's dP^T MMA is
// issued before the dQ drain is awaited and only its S^T MMA waits for it.
// d = 64: dV [0,64) dK [64,128), then per 64-query half h (chunks 2h, 2h+1)
// S^T at 128 + 128h and dP^T 64 columns after it, dQ [384,448). Each P/dS
// warpgroup owns one half: the MMA thread issues the half's next S^T/dP^T
// as soon as it has issued the half's last dV/dK k-steps, so one warpgroup
// works on tile t+1 while the MMAs of the other's half of tile t run.
#pragma once

#include "sm100.cuh"
#include "padmask.cuh"

namespace attn {
namespace bwdtc {

constexpr int kBN = 128;      // keys per work item
constexpr int kBM = 128;      // queries per tile
constexpr int kChunks = 4;    // 32-query chunks of a tile
constexpr int kThreads = 512;
constexpr int kWarpDq = 8;         // first warp of the dQ warpgroup
constexpr int kWarpProducer = 12;
constexpr int kWarpMma = 13;
constexpr int kWarpConv = 14;      // first of the two dQ converter warps
constexpr int kConvWarps = 2;

// Counters in the workspace (int32; all zeroed by the preprocess kernel).
constexpr int kCntSched = 0;        // next work item
constexpr int kCntConvClaim = 1;    // next dQ slab to convert
constexpr int kCntSchedDq = 2;      // next work item of the separate dQ pass
constexpr int kCntHeadBase = 64;    // [BH]: landed work items x 4 per head

// Lane 0 of a warp: wait until *cnt reaches target. Gives up (false) on the
// CTA's abort flag, or when the count has not moved for the time budget (a
// count that keeps moving is a head still being worked on, however long).
__device__ __forceinline__ bool wait_count(const int* cnt, int target, const volatile int* abort,
                                           uint64_t budget_ns) {
    uint64_t t0 = global_timer_ns();
    uint32_t sleep_ns = 128;
    int seen = -1;
    for (int c; (c = ld_acquire_gpu(cnt)) < target;) {
        if (c != seen) {
            seen = c;
            t0 = global_timer_ns();
        } else if (*abort || global_timer_ns() - t0 > budget_ns) {
            return false;
        }
        __nanosleep(sleep_ns);
        if (sleep_ns < 1024) sleep_ns *= 2;
    }
    return true;
}

// Drop one 32-row slab of the accumulator from L2 once converted: its sums
// are dead, and the next call zeroes it again before use, so writing it back
// to HBM would be wasted traffic. D/32 lines per row, one per lane and step.
template <int D>
__device__ __forceinline__ void discard_slab(const float* acc, int bh, int row0, int n, int lane) {
    constexpr int kLinesPerRow = D / 32;
    const size_t base = size_t(bh) * n;
#pragma unroll
    for (int i = 0; i < kLinesPerRow; ++i) {
        const int idx = i * 32 + lane;
        const int r = row0 + idx / kLinesPerRow;
        if (r < n) discard_l2_line(acc + (base + r) * D + (idx % kLinesPerRow) * 32);
    }
}

template <int D>
struct Cfg {
    // At d = 64 the K/V tiles are double-buffered (the next item's load runs
    // during this item), with 3 Q/dO stages; d = 128 has room for neither.
    static constexpr int kKV = (D == 64) ? 2 : 1;
    static constexpr int kStages = (D == 64) ? 3 : 2;
    static constexpr int kPanels = D / 64;
    static constexpr int kTileBytes = 128 * D * 2;     // a 128-row bf16 tile
    static constexpr int kPanelBytes = 128 * 128;      // 128 rows x 128 B
    // d = 64: each P/dS warpgroup runs its own 64-query half of every tile
    // (S^T/dP^T of the half in TMEM columns of its own, signalled on its own
    // barrier), and dQ is staged in a buffer of its own rather than in the dS
    // tile; d = 128 has neither the TMEM nor the shared memory for that.
    static constexpr bool kSplit = (D == 64);
    static constexpr int kOffK = 0;                    // K/V buffer b: K at kOffK + b * kKVBytes,
    static constexpr int kOffV = kOffK + kTileBytes;   // V kTileBytes after it
    static constexpr int kKVBytes = 2 * kTileBytes;
    static constexpr int kOffQ = kKV * kKVBytes;
    static constexpr int kOffdO = kOffQ + kStages * kTileBytes;
    static constexpr int kOffdS = kOffdO + kStages * kTileBytes;   // 128 keys x 128 queries
    // dQ staging, per warp of the dQ warpgroup: 32-row x 32-column fp32
    // buffers (4 KB each, 128B-swizzled) used in turn by the row's D/32
    // segments. d = 128: two per warp, in the dS tile (free between the dQ
    // MMA and the next tile's dS); d = 64: one per warp, after the dS tile.
    static constexpr int kStageBufs = kSplit ? 1 : 2;
    static constexpr int kStageWarpBytes = kStageBufs * 4096;
    static constexpr int kOffStage = kSplit ? kOffdS + 128 * 128 * 2 : kOffdS;
    static constexpr int kOffLse = kSplit ? kOffStage + 4 * kStageWarpBytes : kOffdS + 128 * 128 * 2;
    static constexpr int kOffDd = kOffLse + kStages * kBM * 4;
    static constexpr int kOffBar = kOffDd + kStages * kBM * 4;
    static constexpr int kSmemBytes = kOffBar + 512;
    static constexpr bool kAlias = (D == 128);
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColdV = 0;
    static constexpr uint32_t kColdK = D;
    // S^T and dP^T of the 32-query chunk c (chunks 2h, 2h+1 form half h).
    // bf16 P^T / dS^T are written over the first 16 of the chunk's columns.
    // d = 128: S^T [256,384), dP^T [384,512). d = 64, per half h: S^T at
    // 128 + 128h, dP^T 64 columns after it.
    static constexpr uint32_t col_s(int c) {
        return kSplit ? 2 * D + (c >> 1) * 128 + (c & 1) * 32 : 2 * D + 32 * c;
    }
    static constexpr uint32_t col_dp(int c) { return col_s(c) + (kSplit ? 64 : 128); }
    static constexpr uint32_t kColdQ = kAlias ? 2 * D : 2 * D + 256;
};
static_assert(Cfg<64>::kSmemBytes <= 232448 && Cfg<128>::kSmemBytes <= 232448, "shared memory");

struct Bars {
    uint64_t kv_full[2];
    uint64_t kv_empty[2];   // the item's last MMA has read K_j, V_j of buffer b
    uint64_t q_full[4];
    uint64_t q_empty[4];
    uint64_t s_full[2];     // S^T, dP^T of the tile (d = 64: of half h) are in TMEM
    uint64_t ds_chunk[kChunks];
    uint64_t dq_full;
    uint64_t dq_free;
    uint64_t ds_smem_full;
    uint64_t ds_smem_free;
    uint64_t acc_done;
    uint64_t acc_free;      // the epilogue has read dV, dK out of TMEM
    uint64_t epi_done[4];   // an item's dV, dK staged in stage s and read by the TMA
    uint64_t mma_drain;
    uint64_t sched_full[4];     // work item of slot k published by the producer
    uint64_t sched_empty[4];    // ... and read by the 13 consumers
    int sched_item[4];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier area");

// Sixteen queries (columns q0..q0+15 of a tile) for one key row: P^T and dS^T
// from the S^T / dP^T values in registers. P^T and dS^T are written back to
// TMEM at `pcol` / `dscol` (8 columns each, two bf16 per column); the packed
// dS is also returned in `dk` for the shared-memory tile. MASKED applies the
// causal / key-range mask: columns below `keys_masked_below` get P = 0.
template <bool MASKED>
__device__ __forceinline__ void pds_half(int q0, const uint32_t (&sr)[16], const uint32_t (&pr)[16],
                                         const float* lse_s, const float* dd_s,
                                         int keys_masked_below, float scale, float scale_log2,
                                         uint32_t pcol, uint32_t dscol, uint32_t* dk) {
    uint32_t pk[8];
    // Pairs of queries through the paired fp32 instructions (each half
    // rounded exactly as the scalar one), which halve the FMA-pipe issue.
    const f32x2 sl2 = make_f32x2(scale_log2, scale_log2), sc2 = make_f32x2(scale, scale);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse_s + q0 + 4 * g);
        const float4 d4 = *reinterpret_cast<const float4*>(dd_s + q0 + 4 * g);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = 4 * g + 2 * h;
            const float2 x = split_f32x2(fma_x2(
                make_f32x2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), sl2,
                h ? make_f32x2(-l4.z, -l4.w) : make_f32x2(-l4.x, -l4.y)));
            float p0 = ex2(x.x), p1 = ex2(x.y);
            if (MASKED && (q0 + e) < keys_masked_below) p0 = 0.f;
            if (MASKED && (q0 + e + 1) < keys_masked_below) p1 = 0.f;
            const f32x2 t = fma_x2(make_f32x2(__uint_as_float(pr[e]), __uint_as_float(pr[e + 1])), sc2,
                                   h ? make_f32x2(-d4.z, -d4.w) : make_f32x2(-d4.x, -d4.y));
            const float2 ds = split_f32x2(mul_x2(make_f32x2(p0, p1), t));
            pk[2 * g + h] = pack_bf16x2(p0, p1);
            dk[2 * g + h] = pack_bf16x2(ds.x, ds.y);
        }
    }
    tmem_st8(pcol, pk);
    tmem_st8(dscol, dk);
}

// dS of chunk c for key row r into the shared tile (queries contiguous,
// 128B-swizzled), the dQ MMA's A operand.
template <int D>
__device__ __forceinline__ void store_ds_chunk(uint8_t* sdS, int c, int r, const uint32_t (&dk)[16]) {
    using C = Cfg<D>;
    uint8_t* rowp = sdS + (c >> 1) * C::kPanelBytes + r * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int chunk = ((c & 1) * 4 + q) ^ (r & 7);
        *reinterpret_cast<uint4*>(rowp + chunk * 16) =
            make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
    }
}

// The (head, key tile) of work item `b` in schedule order (see the kernel's
// comment). When causal, the last two groups form one: a group's longest
// items run about as long as the whole group takes on all SMs, so in a last
// group of the usual size they would end well after every other CTA.
__device__ __forceinline__ void cta_tile(int b, int num_kt, int BH, int hg, int causal, int& bh,
                                         int& kt) {
    const int groups = (BH + hg - 1) / hg;
    const int tail_groups = causal ? 2 : 1;
    const int tail_head = groups >= tail_groups ? (groups - tail_groups) * hg : 0;   // last group's first head
    const int tail_item = tail_head * num_kt;
    int head0, heads_here, within;
    if (b < tail_item) {
        head0 = (b / (hg * num_kt)) * hg;
        heads_here = hg;
        within = b % (hg * num_kt);
    } else {
        head0 = tail_head;
        heads_here = BH - tail_head;
        within = b - tail_item;
    }
    kt = within / heads_here;
    bh = head0 + within % heads_here;
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
    cta_tile(b, num_kt, BH, hg, causal, it.bh, kt);
    it.k0 = kt * kBN;
    it.mk = keys_valid(key_len, it.bh, H, m);
    it.first_qt = causal ? kt : 0;
    it.T = (it.k0 >= it.mk) ? 1 : num_qt - it.first_qt;          // >= 1
    return it;
}

// The finished fp32 sums of one 32-row slab (rows row0.., clipped at n) of
// head bh, read from the accumulator and written to dQ in bf16 by one warp:
// D/4 lanes per row, 16 bytes each, sixteen rows' loads in flight per lane
// group (D = 128: the whole slab in two rounds).
template <int D>
__device__ __forceinline__ void convert_slab(const float* acc, __nv_bfloat16* out, int bh, int row0,
                                             int n, int lane) {
    constexpr int kLanesPerRow = D / 4;
    constexpr int kRowsPerIter = 32 / kLanesPerRow;
    constexpr int kIters = 32 / kRowsPerIter;
    constexpr int kBatch = kIters < 16 ? kIters : 16;
    const int sub = lane / kLanesPerRow, c4 = (lane % kLanesPerRow) * 4;
    const size_t base = size_t(bh) * n;
#pragma unroll
    for (int i0 = 0; i0 < kIters; i0 += kBatch) {
        float4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int r = row0 + (i0 + u) * kRowsPerIter + sub;
            v[u] = r < n ? __ldcg(reinterpret_cast<const float4*>(acc + (base + r) * D + c4))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int r = row0 + (i0 + u) * kRowsPerIter + sub;
            if (r < n)
                *reinterpret_cast<uint2*>(out + (base + r) * D + c4) =
                    make_uint2(pack_bf16x2(v[u].x, v[u].y), pack_bf16x2(v[u].z, v[u].w));
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
           const __grid_constant__ CUtensorMap tmdQacc, const __grid_constant__ CUtensorMap tmdK,
           const __grid_constant__ CUtensorMap tmdV, const float* __restrict__ lse2,
           const float* __restrict__ Dd, int* __restrict__ counters, const float* dQacc,
           __nv_bfloat16* __restrict__ dQ, int n_pad, int n, int m, int BH, int head_group,
           int causal, float scale, float scale_log2, const int* __restrict__ key_len, int H,
           unsigned long long budget_ns) {
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
    // tiles and dQ rows in L2); inside a group key-tile major, so the longest
    // items of the group (lowest key tiles, if causal) come first. The
    // producer publishes each item to the other roles through a 4-slot ring
    // in shared memory, one item ahead.
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
        for (int kb = 0; kb < 2; ++kb) {
            mbar_init(&bars->kv_full[kb], 1);
            mbar_init(&bars->kv_empty[kb], 1);
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) mbar_init(&bars->s_full[h], 1);
        for (int c = 0; c < kChunks; ++c) mbar_init(&bars->ds_chunk[c], 128);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_free, 128);
        // d = 64: the dQ warpgroup's "dQ read out of TMEM" arrives here too,
        // so one wait covers both conditions of the next dQ MMA.
        mbar_init(&bars->ds_smem_full, C::kSplit ? 256 + 128 : 256);
        mbar_init(&bars->ds_smem_free, 128);
        mbar_init(&bars->acc_done, 1);
        mbar_init(&bars->acc_free, 128);
        for (int s = 0; s < 4; ++s) mbar_init(&bars->epi_done[s], 128);
        mbar_init(&bars->mma_drain, 1);
        for (int k = 0; k < 4; ++k) {
            mbar_init(&bars->sched_full[k], 1);
            mbar_init(&bars->sched_empty[k], 1 + 8 + 4);
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
    // Launched as a programmatic dependent of the preprocess kernel (its
    // CTAs start on an SM once the preprocess CTAs there have left); its
    // outputs (LSE_2, D, the zeroed accumulator and counters) are touched
    // only after this.
    grid_dependency_wait();

    // dQ conversion, by one warp: slabs of 32 rows in head order (the order in
    // which heads finish). Claim a slab, wait until every work item of its
    // head has landed its partials (4 counts per item, one per dQ warp),
    // convert it, drop its fp32 lines; until no slab is left.
    auto convert_loop = [&]() {
        const int units = BH * num_qt * 4;
        const int target = 4 * num_kt;
        for (;;) {
            int u = 0;
            if (lane == 0) u = atomicAdd(counters + kCntConvClaim, 1);
            u = __shfl_sync(0xffffffffu, u, 0);
            if (u >= units) return;
            const int bh = u / (num_qt * 4);
            const int row0 = (u % (num_qt * 4)) * 32;
            int ready = 1;
            if (lane == 0) ready = wait_count(counters + kCntHeadBase + bh, target, abort_flag, budget_ns);
            if (!__shfl_sync(0xffffffffu, ready, 0)) {
                if (lane == 0) {
                    record_device_error(kErrTimeout);
                    *abort_flag = 1;
                }
                return;
            }
            if (row0 < n) {
                convert_slab<D>(dQacc, dQ, bh, row0, n, lane);
                __syncwarp();
                discard_slab<D>(dQacc, bh, row0, n, lane);
            }
        }
    };

    if (!aborted_early && warp == kWarpProducer && lane == 0) {
        // ------------------------------------------------ TMA producer
        prefetch_tensor_map(&tmQ);
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        prefetch_tensor_map(&tmdO);
        prefetch_tensor_map(&tmdQacc);
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
            const int kb = j % C::kKV;
            if (j >= C::kKV &&
                !mbar_wait(&bars->kv_empty[kb], (j / C::kKV - 1) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            mbar_arrive_expect_tx(&bars->kv_full[kb], 2 * C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p) {
                tma_load_3d(smem + C::kOffK + kb * C::kKVBytes + p * C::kPanelBytes, &tmK,
                            &bars->kv_full[kb], p * 64, it.k0, it.bh);
                tma_load_3d(smem + C::kOffV + kb * C::kKVBytes + p * C::kPanelBytes, &tmV,
                            &bars->kv_full[kb], p * 64, it.k0, it.bh);
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
            int nb = G + atomicAdd(counters + kCntSched, 1);
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
        // older than the last stage's worth (and K/V before the last buffer's
        // worth) were consumed, so they have landed.
        for (int i = (kv_issued > C::kKV ? kv_issued - C::kKV : 0); i < kv_issued; ++i)
            (void)mbar_wait_timed(&bars->kv_full[i % C::kKV], (i / C::kKV) & 1, budget_ns);
        for (int t = (g > C::kStages ? g - C::kStages : 0); t < g; ++t)
            (void)mbar_wait_timed(&bars->q_full[t % C::kStages], (t / C::kStages) & 1, budget_ns);
    } else if (!aborted_early && warp == kWarpMma) {
        // ------------------------------------------------ MMA issuer
        // The whole warp walks the loop (waits are warp-wide) and one elected
        // lane issues the MMAs and commits.
        const uint32_t leader = elect_leader();
        constexpr uint32_t idSP = idesc_bf16_f32(kBN, kBM, 0, 0);       // S^T, dP^T
        constexpr uint32_t idHalf = idesc_bf16_f32(kBN, kBM / 2, 0, 0); // ... of a 64-query half
        constexpr uint32_t idKV = idesc_bf16_f32(kBN, D, 0, 1);         // dV, dK
        constexpr uint32_t idQ = idesc_bf16_f32(kBM, D, 1, 1);          // dQ
        uint32_t sK = smem_addr(smem + C::kOffK), sV = smem_addr(smem + C::kOffV);   // per item
        const uint32_t sdS = smem_addr(smem + C::kOffdS);
        // dP^T(g) = V dO(g)^T once Q/dO(g) are in; its columns are free once
        // the previous tile's dK MMAs (issued earlier) have read dS^T.
        auto issue_dP = [&](int g) -> bool {
            const int s = g % C::kStages;
            if (!mbar_wait_warp(&bars->q_full[s], (g / C::kStages) & 1, abort_flag, budget_ns)) return false;
            tc_fence_after();
            const uint64_t aV = sdesc_sw128(sV, 16, 1024);
            const uint64_t bdO = sdesc_sw128(smem_addr(smem + C::kOffdO + s * C::kTileBytes), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::col_dp(0), sdesc_adv(aV, koff), sdesc_adv(bdO, koff), idSP, kk > 0,
                         leader);
            }
            return true;
        };
        // S^T(g) = K Q(g)^T (issued after dP^T(g)); s_full then reports both.
        // At d = 128 its columns hold the previous tile's dQ until the dQ
        // warpgroup has read it out.
        auto issue_S = [&](int g) -> bool {
            if (C::kAlias && g > 0 &&
                !mbar_wait_warp(&bars->dq_free, (g - 1) & 1, abort_flag, budget_ns))
                return false;
            tc_fence_after();
            const uint64_t aK = sdesc_sw128(sK, 16, 1024);
            const uint64_t bQ =
                sdesc_sw128(smem_addr(smem + C::kOffQ + (g % C::kStages) * C::kTileBytes), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::col_s(0), sdesc_adv(aK, koff), sdesc_adv(bQ, koff), idSP, kk > 0, leader);
            }
            mma_commit_w(&bars->s_full[0], leader);
            return true;
        };
        // d = 64: dP^T and S^T of the 64-query half h of tile g (queries
        // 64h.., rows 64h.. of the Q/dO tiles, 8 KB in); s_full[h] reports
        // both. Their columns were last read by the half's dV/dK MMAs of the
        // previous tile, issued earlier.
        auto issue_half = [&](int g, int h) -> bool {
            const int s = g % C::kStages;
            // Half 1 always follows half 0 of the same tile, whose wait saw Q/dO in.
            if (h == 0 && !mbar_wait_warp(&bars->q_full[s], (g / C::kStages) & 1, abort_flag, budget_ns))
                return false;
            tc_fence_after();
            const uint64_t bQh = sdesc_sw128(smem_addr(smem + C::kOffQ + s * C::kTileBytes) + h * 8192, 16, 1024);
            const uint64_t bdOh = sdesc_sw128(smem_addr(smem + C::kOffdO + s * C::kTileBytes) + h * 8192, 16, 1024);
            const uint64_t aV = sdesc_sw128(sV, 16, 1024), aK = sdesc_sw128(sK, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::col_dp(2 * h), sdesc_adv(aV, koff), sdesc_adv(bdOh, koff), idHalf, kk > 0,
                         leader);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss_w(tmem + C::col_s(2 * h), sdesc_adv(aK, koff), sdesc_adv(bQh, koff), idHalf, kk > 0,
                         leader);
            }
            mma_commit_w(&bars->s_full[h], leader);
            return true;
        };
        bool ok = true;
        int g = 0;
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const int T = item(b).T;
            const int kb = j % C::kKV;
            if (!mbar_wait_warp(&bars->kv_full[kb], (j / C::kKV) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            sK = smem_addr(smem + C::kOffK + kb * C::kKVBytes);
            sV = smem_addr(smem + C::kOffV + kb * C::kKVBytes);
            // d = 128: per tile dP^T, S^T, the dV/dK k-steps chunk by chunk,
            // then dQ; the next tile's S^T overwrites dQ's columns, so it waits
            // for the dQ warpgroup to read them out. d = 64: each half's next
            // dP^T/S^T is issued as soon as the half's last dV/dK k-steps are,
            // so a P/dS warpgroup starts on its half of tile t+1 while the
            // other warpgroup still works on tile t.
            if (C::kSplit && (!issue_half(g, 0) || !issue_half(g, 1))) { ok = false; break; }
            for (int t = 0; t < T; ++t, ++g) {
                const int s = g % C::kStages;
                const uint32_t sQ = smem_addr(smem + C::kOffQ + s * C::kTileBytes);
                const uint32_t sdO = smem_addr(smem + C::kOffdO + s * C::kTileBytes);
                if (!C::kSplit && (!issue_dP(g) || !issue_S(g))) { ok = false; break; }
                // The item's first dV/dK MMAs overwrite the accumulators: the
                // previous item's epilogue must have read them out.
                if (t == 0 && j > 0 &&
                    !mbar_wait_warp(&bars->acc_free, (j - 1) & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                // dV += P^T dO and dK += dS^T Q, two k-steps per 32-query chunk.
                // d = 128: chunk by chunk as soon as a P/dS warpgroup has written
                // it; the two warpgroups finish chunks 0 and 2 first, then 1
                // and 3. d = 64: a half at a time (its warpgroup signals chunk
                // 2h+1 after chunk 2h), then the half's next S^T/dP^T.
                bool first = (t == 0);
                const uint64_t bdO = sdesc_sw128(sdO, C::kPanelBytes, 1024);
                const uint64_t bQ = sdesc_sw128(sQ, C::kPanelBytes, 1024);
                auto issue_chunk = [&](int c) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int kk = 2 * c + h;                      // queries 16kk..16kk+15
                        mma_ts_w(tmem + C::kColdV, tmem + C::col_s(c) + 8 * h, sdesc_adv(bdO, kk * 2048), idKV,
                                 !first, leader);
                        mma_ts_w(tmem + C::kColdK, tmem + C::col_dp(c) + 8 * h, sdesc_adv(bQ, kk * 2048), idKV,
                                 !first, leader);
                        first = false;
                    }
                };
                if (C::kSplit) {
                    for (int h = 0; h < 2; ++h) {
                        if (!mbar_wait_warp(&bars->ds_chunk[2 * h + 1], g & 1, abort_flag, budget_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_chunk(2 * h);
                        issue_chunk(2 * h + 1);
                        if (t + 1 < T && !issue_half(g + 1, h)) {
                            ok = false;
                            break;
                        }
                    }
                } else {
                    for (int ci = 0; ci < kChunks; ++ci) {
                        const int c = (ci >> 1) | ((ci & 1) << 1);    // 0, 2, 1, 3
                        if (!mbar_wait_warp(&bars->ds_chunk[c], g & 1, abort_flag, budget_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_chunk(c);
                    }
                }
                if (!ok) break;
                mma_commit_w(&bars->q_empty[s], leader);
                if (t == T - 1) mma_commit_w(&bars->acc_done, leader);
                // dS(g) in shared memory (and, d = 64, dQ(g-1) read out of TMEM).
                if (!mbar_wait_warp(&bars->ds_smem_full, g & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t aS = sdesc_sw128(sdS, C::kPanelBytes, 1024);
                const uint64_t bK = sdesc_sw128(sK, C::kPanelBytes, 1024);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ss_w(tmem + C::kColdQ, sdesc_adv(aS, kk * 2048), sdesc_adv(bK, kk * 2048), idQ, kk > 0,
                             leader);
                mma_commit_w(&bars->dq_full, leader);
                // The item's last MMA has been issued: K_j, V_j are free once
                // it has completed.
                if (t == T - 1) mma_commit_w(&bars->kv_empty[kb], leader);
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
        uint8_t* sdS = smem + C::kOffdS;
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
                    !mbar_wait_warp(&bars->s_full[C::kSplit ? grp : 0], g & 1, abort_flag, budget_ns)) {
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
                // Four half-chunks of 16 queries (two chunks), each half's TMEM
                // loads issued while the previous half is computed. A chunk's
                // P^T/dS^T go into the first 16 of its own 32 columns: half h
                // of chunk c writes columns 32c+8h..32c+8h+7, which it has read.
                uint32_t ds0[16], ds1[16];
                uint32_t sA[16], pA[16], sB[16], pB[16];
                const int cbase = 2 * grp;
                tmem_ld16(tl + C::col_s(cbase), sA);
                tmem_ld16(tl + C::col_dp(cbase), pA);
                tmem_ld_wait();
#pragma unroll
                for (int hc = 0; hc < 4; ++hc) {
                    const int c = cbase + (hc >> 1), half = hc & 1;
                    const int qcol = 32 * c + 16 * half;              // first query of the half
                    uint32_t (&scur)[16] = (hc & 1) ? sB : sA;
                    uint32_t (&pcur)[16] = (hc & 1) ? pB : pA;
                    uint32_t (&snxt)[16] = (hc & 1) ? sA : sB;
                    uint32_t (&pnxt)[16] = (hc & 1) ? pA : pB;
                    if (hc < 3) {
                        const int cn = cbase + ((hc + 1) >> 1), hn = (hc + 1) & 1;
                        tmem_ld16(tl + C::col_s(cn) + 16 * hn, snxt);
                        tmem_ld16(tl + C::col_dp(cn) + 16 * hn, pnxt);
                    }
                    uint32_t* dk = ((hc >> 1) ? ds1 : ds0) + 8 * half;
                    const uint32_t pcol = tl + C::col_s(c) + 8 * half;
                    const uint32_t dscol = tl + C::col_dp(c) + 8 * half;
                    if (masked)
                        pds_half<true>(qcol, scur, pcur, lse_s, dd_s, below, scale, scale_log2, pcol,
                                       dscol, dk);
                    else
                        pds_half<false>(qcol, scur, pcur, lse_s, dd_s, below, scale, scale_log2, pcol,
                                        dscol, dk);
                    if (half == 1) {
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(&bars->ds_chunk[c]);
                    }
                    if (hc < 3) tmem_ld_wait();
                }
                // d = 128: the dS tile doubles as the dQ warpgroup's staging
                // buffer for the previous tile: write it once the TMA has read
                // that. d = 64: once the previous tile's dQ MMA has read it.
                if (g > 0 && !(C::kSplit ? mbar_wait_warp(&bars->dq_full, (g - 1) & 1, abort_flag, budget_ns)
                                         : mbar_wait_warp(&bars->ds_smem_free, (g - 1) & 1, abort_flag,
                                                          budget_ns))) {
                    ok = false;
                    break;
                }
                store_ds_chunk<D>(sdS, 2 * grp, r, ds0);
                store_ds_chunk<D>(sdS, 2 * grp + 1, r, ds1);
                fence_proxy_async_smem();
                mbar_arrive(&bars->ds_smem_full);
            }
            if (!ok) break;
            // The item's dV/dK epilogue is the dQ warpgroup's: this group goes
            // straight on to the next item.
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
    } else if (!aborted_early && warp >= kWarpDq && warp < kWarpDq + 4) {
        // ------------------------------------------------ dQ warpgroup
        // Thread r owns query row r of the tile (its TMEM lane). Each warp
        // stages its 32 rows one 32-column segment at a time, in the 128-byte
        // swizzled layout of the accumulator's tensor map, and one lane hands
        // each segment to the TMA engine as a tiled reduce-add; rows past n
        // are clipped by the TMA. d = 128 stages in the dS tile, free from
        // the dQ MMA's completion until the P/dS warpgroups write the next
        // tile's dS; d = 64 in a buffer of its own.
        const int wq = warp & 3;
        const uint32_t tl = tmem + (uint32_t(wq * 32) << 16);
        uint8_t* stage = smem + C::kOffStage + wq * C::kStageWarpBytes;
        // d = 64: "dQ read out" goes to the barrier of the next dQ MMA, which
        // also counts the dS stores; the first dQ MMA has nothing to wait for.
        uint64_t* dq_read = C::kSplit ? &bars->ds_smem_full : &bars->dq_free;
        if (C::kSplit) mbar_arrive(dq_read);
        bool ok = true;
        int g = 0;
        for (int j = 0; ok; ++j) {
            const int b = next_item(j, true);
            if (b == -1) break;
            if (b < 0) { ok = false; break; }
            const Item it = item(b);
            for (int t = 0; t < it.T; ++t, ++g) {
                const int row0 = (it.first_qt + t) * kBM + wq * 32;
                if (!mbar_wait_warp(&bars->dq_full, g & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // 32 columns (one segment) at a time through two register
                // buffers: segment sg + 2 is loaded from TMEM as soon as
                // segment sg has been written to shared memory, so the loads
                // overlap the staging and the TMEM columns are released
                // (dq_free) as soon as the last segment is in registers.
                constexpr int kSegs = D / 32;
                uint32_t va[32], vb[32];
                tmem_ld32(tl + C::kColdQ, va);
                tmem_ld32(tl + C::kColdQ + 32, vb);
                tmem_ld_wait();
                if (kSegs == 2) {
                    tc_fence_before();
                    mbar_arrive(dq_read);
                }
#pragma unroll
                for (int sg = 0; sg < kSegs; ++sg) {                  // columns 32sg..32sg+31
                    uint32_t (&v)[32] = (sg & 1) ? vb : va;
                    uint8_t* buf = stage + (sg % C::kStageBufs) * 4096;
                    if (sg >= C::kStageBufs) {
                        if (lane == 0) {                              // buffer's previous segment read
                            if (C::kStageBufs == 2) bulk_wait_group_read1();
                            else bulk_wait_group_read0();
                        }
                        __syncwarp();
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        *reinterpret_cast<uint4*>(buf + lane * 128 + ((k ^ (lane & 7)) * 16)) =
                            make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                    if (sg + 2 < kSegs) {
                        tmem_ld32(tl + C::kColdQ + 32 * (sg + 2), v);
                        if (sg + 3 == kSegs) {
                            tmem_ld_wait();
                            tc_fence_before();
                            mbar_arrive(dq_read);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_reduce_add_3d(&tmdQacc, buf, 32 * sg, row0, it.bh);
                        bulk_commit_group();
                    }
                }
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
                if (!C::kSplit) mbar_arrive(&bars->ds_smem_free);
            }
            if (!ok) break;
            // Epilogue of item j: dV and dK, staged in the Q / dO halves of
            // the stage that held the item's last tile (every MMA that read it
            // is complete once acc_done has fired; the producer reloads it
            // only after epi_done). Each thread reads its key row out of TMEM
            // 32 columns at a time, converts it to bf16 and stages it in the
            // 128-byte swizzled layout of the output's tensor map; one lane per
            // warp stores 32 x 64 boxes with the TMA (rows past m clipped).
            // The accumulators are released for the next item as soon as they
            // have been read. Done here rather than by the P/dS warpgroups, so
            // that they start on the next item at once.
            if (!mbar_wait_warp(&bars->acc_done, j & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                const int s_last = (g - 1) % C::kStages;
#pragma unroll
                for (int which = 0; which < 2; ++which) {             // dV, then dK
                    const uint32_t col = which == 0 ? C::kColdV : C::kColdK;
                    uint8_t* st = smem + (which == 0 ? C::kOffQ : C::kOffdO) + s_last * C::kTileBytes +
                                  wq * (32 * D * 2);
#pragma unroll
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t rr[32];
                        tmem_ld32(tl + col + 32 * q, rr);
                        tmem_ld_wait(rr);
                        uint8_t* buf = st + (q >> 1) * 4096;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int kc = 4 * (q & 1) + k;        // 16-byte chunk of the 128-byte row
                            *reinterpret_cast<uint4*>(buf + lane * 128 + ((kc ^ (lane & 7)) * 16)) = make_uint4(
                                pack_bf16x2(__uint_as_float(rr[8 * k + 0]), __uint_as_float(rr[8 * k + 1])),
                                pack_bf16x2(__uint_as_float(rr[8 * k + 2]), __uint_as_float(rr[8 * k + 3])),
                                pack_bf16x2(__uint_as_float(rr[8 * k + 4]), __uint_as_float(rr[8 * k + 5])),
                                pack_bf16x2(__uint_as_float(rr[8 * k + 6]), __uint_as_float(rr[8 * k + 7])));
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->acc_free);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int which = 0; which < 2; ++which) {
                        uint8_t* st = smem + (which == 0 ? C::kOffQ : C::kOffdO) + s_last * C::kTileBytes +
                                      wq * (32 * D * 2);
#pragma unroll
                        for (int pnl = 0; pnl < C::kPanels; ++pnl)
                            tma_store_3d(which == 0 ? &tmdV : &tmdK, st + pnl * 4096, 64 * pnl,
                                         it.k0 + 32 * wq, it.bh);
                    }
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
                __syncwarp();
                mbar_arrive(&bars->epi_done[s_last]);
            }
            // Every partial of this item has been handed to the TMA: once they
            // have landed, count the item for its head (the converter warps
            // wait for that count). The next item's first dQ is microseconds
            // away (its K/V load and first tile come first), so this wait is
            // off the pipeline's path.
            if (lane == 0) {
                bulk_wait_group0();
                fence_proxy_async_global();
                red_add_release_gpu(counters + kCntHeadBase + it.bh, 1);
            }
            __syncwarp();
        }
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
    } else if (!aborted_early && warp >= kWarpConv && warp < kWarpConv + kConvWarps) {
        // ------------------------------------------------ dQ converters
        convert_loop();
    }
    // A warp whose own work has run out helps with the conversion: at the end
    // of the launch the last heads finish together, and two warps per CTA
    // would take several rounds of slabs for them.
    __syncwarp();
    if (!aborted_early && warp < kWarpConv && *abort_flag == 0) convert_loop();

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace bwdtc
}  // namespace attn
