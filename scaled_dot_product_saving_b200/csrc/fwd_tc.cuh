// fwd_tc.cuh -- tensor-core forward for bf16, d == dv in {64, 128}.
//
// Computes O = softmax(scale * Q K^T) V and the row log-sum-exp (the forward
// whose softmax statistics the backward recomputes P from: "Attention Backward
// Pass (dQ, dK, dV)", section on the forward; under the causal mask key j > i
// is excluded before the softmax).
//
// One CTA computes two adjacent 128-row query tiles, A = 2p and B = 2p + 1,
// of one (batch, head), sharing every key and value tile it loads; under the
// causal mask B needs one key tile more than A. CTAs run in groups of heads
// (so a group's keys and values stay in L2), heaviest query rows first within
// a group. For each 128-key tile t and each query tile x:
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
// Shared memory: Q_A, Q_B, then K and V rings with their own barriers (a K
// tile is released as soon as both S products that read it are done).
#pragma once

#include "sm100.cuh"

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
    static constexpr int kSmemBytes = kOffBar + 256;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0;                // S_x at kColS0 + 128 x
    static constexpr uint32_t kColO0 = 256;              // O_x at kColO0 + D x
    static constexpr int kStageWarpBytes = 32 * D * 2;  // epilogue: 32 rows per warp
};
static_assert(Cfg<128>::kSmemBytes <= 232448, "shared memory");

struct Bars {
    uint64_t q_full;
    uint64_t k_full[4];
    uint64_t k_empty[4];
    uint64_t v_full[4];
    uint64_t v_empty[4];
    uint64_t s_full[2];
    uint64_t p_half[2];   // P of keys 0..63 of the tile written
    uint64_t p_full[2];   // all of P written
    uint64_t o_done[2];
    uint64_t mma_drain;
    uint32_t tmem_base;
    int abort;
};

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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
           float* __restrict__ LSE, int n, int m, int BH, int head_group, int causal,
           float scale_log2, unsigned long long budget_ns) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_qt = (n + kBM - 1) / kBM;
    const int num_pairs = (num_qt + 1) / 2;
    int bh, pair;
    cta_pair(int(blockIdx.x), num_pairs, BH, head_group, bh, pair);
    const int num_kt = (m + kBN - 1) / kBN;
    const bool has_b = 2 * pair + 1 < num_qt;
    // query tile and number of key tiles of tile A (x = 0) and tile B (x = 1)
    const int qt_a = 2 * pair, qt_b = 2 * pair + 1;
    const int nkv_a = causal ? min(num_kt, qt_a + 1) : num_kt;
    const int nkv_b = has_b ? (causal ? min(num_kt, qt_b + 1) : num_kt) : 0;
    auto qt_of = [&](int x) { return x ? qt_b : qt_a; };
    auto nkv_of = [&](int x) { return x ? nkv_b : nkv_a; };
    const int num_kv = max(nkv_a, nkv_b);

    if (threadIdx.x == 0) {
        // The swizzled tiles need a 1024-byte aligned base. A CTA that starts
        // after another one gave up a wait does no work at all.
        const bool misaligned = (smem_addr(smem) & 1023u) != 0;
        if (misaligned) record_device_error(kErrTimeout);
        bars->abort = (misaligned || *reinterpret_cast<volatile unsigned int*>(&g_device_error) != 0) ? 1 : 0;
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->p_half[x], 128);
            mbar_init(&bars->p_full[x], 128);
            mbar_init(&bars->o_done[x], 1);
        }
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
        const int nq = has_b ? 2 : 1;
        mbar_arrive_expect_tx(&bars->q_full, nq * C::kTileBytes);
        for (int x = 0; x < nq; ++x)
            for (int p = 0; p < C::kPanels; ++p)
                tma_load_3d(smem + C::kOffQ + x * C::kTileBytes + p * C::kPanelBytes, &tmQ,
                            &bars->q_full, p * 64, qt_of(x) * kBM, bh);
        int k_issued = 0, v_issued = 0;
        for (int t = 0; t < num_kv; ++t) {
            const int sk = t % C::kKStages, sv = t % C::kVStages;
            if (t >= C::kKStages &&
                !mbar_wait(&bars->k_empty[sk], (t / C::kKStages - 1) & 1, abort_flag, budget_ns))
                break;
            mbar_arrive_expect_tx(&bars->k_full[sk], C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p)
                tma_load_3d(smem + C::kOffK + sk * C::kTileBytes + p * C::kPanelBytes, &tmK,
                            &bars->k_full[sk], p * 64, t * kBN, bh);
            ++k_issued;
            if (t >= C::kVStages &&
                !mbar_wait(&bars->v_empty[sv], (t / C::kVStages - 1) & 1, abort_flag, budget_ns))
                break;
            mbar_arrive_expect_tx(&bars->v_full[sv], C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p)
                tma_load_3d(smem + C::kOffV + sv * C::kTileBytes + p * C::kPanelBytes, &tmV,
                            &bars->v_full[sv], p * 64, t * kBN, bh);
            ++v_issued;
        }
        if (v_issued < num_kv) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: every load issued must land before the CTA may exit. Tiles
        // older than the last ring's worth were consumed, so they have landed.
        (void)mbar_wait_timed(&bars->q_full, 0, budget_ns);
        for (int t = (k_issued > C::kKStages ? k_issued - C::kKStages : 0); t < k_issued; ++t)
            (void)mbar_wait_timed(&bars->k_full[t % C::kKStages], (t / C::kKStages) & 1, budget_ns);
        for (int t = (v_issued > C::kVStages ? v_issued - C::kVStages : 0); t < v_issued; ++t)
            (void)mbar_wait_timed(&bars->v_full[t % C::kVStages], (t / C::kVStages) & 1, budget_ns);
    } else if (!aborted_early && warp == kWarpMma && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, 0, 0);
        constexpr uint32_t idO = idesc_bf16_f32(kBM, D, 0, 1);
        auto issue_S = [&](int x, int t) {
            const uint32_t sQ = smem_addr(smem + C::kOffQ + x * C::kTileBytes);
            const uint32_t sK = smem_addr(smem + C::kOffK + (t % C::kKStages) * C::kTileBytes);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss(tmem + C::kColS0 + 128 * x, sdesc_sw128(sQ + koff, 16, 1024),
                       sdesc_sw128(sK + koff, 16, 1024), idS, kk > 0);
            }
            mma_commit(&bars->s_full[x]);
        };
        // O_x += P_x V_t over keys 64h .. 64h+63 of the tile
        auto issue_PV = [&](int x, int t, int h) {
            const uint32_t sV = smem_addr(smem + C::kOffV + (t % C::kVStages) * C::kTileBytes);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int kk = 4 * h + k4;
                mma_ts(tmem + C::kColO0 + D * x, tmem + C::kColS0 + 128 * x + kk * 8,
                       sdesc_sw128(sV + kk * 2048, C::kPanelBytes, 1024), idO, (t > 0 || kk > 0));
            }
        };
        bool ok = mbar_wait(&bars->q_full, 0, abort_flag, budget_ns) &&
                  mbar_wait(&bars->k_full[0], 0, abort_flag, budget_ns);
        if (ok) {
            tc_fence_after();
            for (int x = 0; x < 2; ++x)
                if (nkv_of(x) > 0) issue_S(x, 0);
            mma_commit(&bars->k_empty[0]);
        }
        for (int t = 0; ok && t < num_kv; ++t) {
            bool v_ready = false, k_ready = false;
            for (int x = 0; x < 2; ++x) {
                if (t >= nkv_of(x)) continue;
                if (!mbar_wait(&bars->p_half[x], t & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                if (!v_ready) {
                    if (!mbar_wait(&bars->v_full[t % C::kVStages], (t / C::kVStages) & 1,
                                   abort_flag, budget_ns)) {
                        ok = false;
                        break;
                    }
                    v_ready = true;
                }
                tc_fence_after();
                issue_PV(x, t, 0);
                if (!mbar_wait(&bars->p_full[x], t & 1, abort_flag, budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_PV(x, t, 1);
                if (t + 1 < nkv_of(x)) {
                    if (!k_ready) {
                        const int t1 = t + 1;
                        if (!mbar_wait(&bars->k_full[t1 % C::kKStages], (t1 / C::kKStages) & 1,
                                       abort_flag, budget_ns)) {
                            ok = false;
                            break;
                        }
                        k_ready = true;
                        tc_fence_after();
                    }
                    issue_S(x, t + 1);
                } else {
                    mma_commit(&bars->o_done[x]);   // last product into O_x
                }
            }
            if (!ok) break;
            if (k_ready) mma_commit(&bars->k_empty[(t + 1) % C::kKStages]);
            mma_commit(&bars->v_empty[t % C::kVStages]);
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: all MMAs issued here complete before TMEM is released.
        mma_commit(&bars->mma_drain);
        (void)mbar_wait_timed(&bars->mma_drain, 0, budget_ns);
    } else if (!aborted_early && warp < 8) {
        // ------------------------------------------------ softmax warpgroups
        const int x = warp >> 2;                         // query tile A or B
        const int r = threadIdx.x & 127;                 // row in the tile == TMEM lane
        const uint32_t tl = tmem + (uint32_t((warp & 3) * 32) << 16);
        const uint32_t tS = tl + C::kColS0 + 128 * x, tO = tl + C::kColO0 + D * x;
        const int q0 = qt_of(x) * kBM;
        const int row = q0 + r;
        const int ntile = nkv_of(x);
        const bool neg = scale_log2 < 0.f;
        const f32x2 sl2 = make_f32x2(scale_log2, scale_log2);
        // Keys after kmax are masked: past the end, or after the row (causal).
        const int kmax = causal ? min(row, m - 1) : m - 1;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < ntile; ++t) {
            if (!mbar_wait_warp(&bars->s_full[x], t & 1, abort_flag, budget_ns)) {
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
        }
        if (ok && ntile > 0 && !mbar_wait_warp(&bars->o_done[x], 0, abort_flag, budget_ns))
            ok = false;
        if (ok && ntile > 0) {
            // Epilogue: O / sum as bf16, staged per warp (32 rows) in the
            // 128B-swizzled layout of O's tensor map inside this tile's Q buffer
            // (no MMA reads it any more), stored with the TMA; rows past n are
            // clipped by the tensor map. LSE in natural log.
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
                    tma_store_3d(&tmO, buf, 64 * pnl, q0 + 32 * (warp & 3), bh);
                    bulk_commit_group();
                }
            }
            if (row < n) LSE[size_t(bh) * n + row] = (m_run + log2f(l_run)) * kLn2;
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
        } else if (!ok) {
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
