// fwd_tc.cuh -- tensor-core forward for bf16, d == dv in {64, 128}.
//
// One CTA computes a 128-row query tile of one (batch, head) and walks the
// key/value tiles (128 keys each; only tiles at or below the diagonal when
// causal):
//   S = Q K_t^T                     tcgen05.mma, A = Q, B = K_t (both K-major
//                                   in shared memory), fp32 D in TMEM
//   running max / sum, P = 2^(S*scale*log2e - max)   128 softmax threads,
//                                   one query row (TMEM lane) each
//   O += P V_t                      tcgen05.mma, A = P read from TMEM (bf16
//                                   written over its own S columns),
//                                   B = V_t (MN-major), O in TMEM
// At the end O / sum goes to global memory as bf16 and the row's log-sum-exp
// (natural log) as fp32. The running max is only raised, and O rescaled, when
// a new row max exceeds the one in use by more than 2^8 in P.
//
// Warp roles (256 threads): warp 0 = TMA producer, warp 1 = TMEM allocator
// and MMA issuer, warps 4-7 = softmax (warp 4+w owns TMEM lanes 32w..32w+31).
// S is double-buffered in TMEM so that the tensor cores compute S_{t+1}
// while the softmax threads work on S_t.
#pragma once

#include "sm100.cuh"

namespace attn {
namespace fwdtc {

constexpr int kBM = 128;      // queries per CTA
constexpr int kBN = 128;      // keys per tile
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
    static constexpr int kStages = (D == 64) ? 4 : 2;
    static constexpr int kPanels = D / 64;              // 64-column swizzle panels
    static constexpr int kTileBytes = kBM * D * 2;      // a 128-row bf16 tile
    static constexpr int kPanelBytes = kBM * 128;       // 128 rows x 128 B
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kBarBytes = 256;
    static constexpr int kSmemBytes = kOffBar + kBarBytes;
    // TMEM columns (512 allocated): two S buffers of 128 fp32 columns, then O.
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
};

struct Bars {
    uint64_t q_full;
    uint64_t kv_full[4];
    uint64_t kv_empty[4];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done;
    uint64_t mma_drain;
    uint32_t tmem_base;
    int abort;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
           float* __restrict__ LSE, int n, int m, int BH, int causal, float scale_log2,
           unsigned long long budget_ns) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_qt = (n + kBM - 1) / kBM;
    const int qt = num_qt - 1 - int(blockIdx.x / BH);   // heaviest (last) query tiles first
    const int bh = int(blockIdx.x % BH);
    const int q0 = qt * kBM;
    const int kv_end = causal ? min(m, q0 + kBM) : m;
    const int num_kv = (kv_end + kBN - 1) / kBN;

    if (threadIdx.x == 0) {
        // The swizzled tiles need a 1024-byte aligned base. A CTA that starts
        // after another one gave up a wait does no work at all.
        const bool misaligned = (smem_addr(smem) & 1023u) != 0;
        if (misaligned) record_device_error(kErrTimeout);
        bars->abort = (misaligned || *reinterpret_cast<volatile unsigned int*>(&g_device_error) != 0) ? 1 : 0;
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->p_full[b], 128);
        }
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->mma_drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const bool aborted_early = bars->abort != 0;

    if (!aborted_early && warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        prefetch_tensor_map(&tmQ);
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        mbar_arrive_expect_tx(&bars->q_full, C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
            tma_load_3d(smem + C::kOffQ + p * C::kPanelBytes, &tmQ, &bars->q_full, p * 64, q0, bh);
        int issued = 0;
        for (int t = 0; t < num_kv; ++t) {
            const int s = t % C::kStages, k = t / C::kStages;
            if (t >= C::kStages &&
                !mbar_wait(&bars->kv_empty[s], (k - 1) & 1, abort_flag, budget_ns)) {
                record_device_error(kErrTimeout);
                *abort_flag = 1;
                break;
            }
            mbar_arrive_expect_tx(&bars->kv_full[s], 2 * C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p) {
                tma_load_3d(smem + C::kOffK + s * C::kTileBytes + p * C::kPanelBytes, &tmK,
                            &bars->kv_full[s], p * 64, t * kBN, bh);
                tma_load_3d(smem + C::kOffV + s * C::kTileBytes + p * C::kPanelBytes, &tmV,
                            &bars->kv_full[s], p * 64, t * kBN, bh);
            }
            ++issued;
        }
        // Drain: every load issued must land before the CTA may exit. Tiles
        // older than the last kStages were consumed, so they have landed.
        (void)mbar_wait_timed(&bars->q_full, 0, budget_ns);
        for (int t = (issued > C::kStages ? issued - C::kStages : 0); t < issued; ++t)
            (void)mbar_wait_timed(&bars->kv_full[t % C::kStages], (t / C::kStages) & 1, budget_ns);
    } else if (!aborted_early && warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, 0, 0);
        constexpr uint32_t idO = idesc_bf16_f32(kBM, D, 0, 1);
        const uint32_t sQ = smem_addr(smem + C::kOffQ);
        bool ok = mbar_wait(&bars->q_full, 0, abort_flag, budget_ns);
        auto issue_S = [&](int t) -> bool {
            const int s = t % C::kStages;
            if (!mbar_wait(&bars->kv_full[s], (t / C::kStages) & 1, abort_flag, budget_ns))
                return false;
            tc_fence_after();
            const uint32_t sK = smem_addr(smem + C::kOffK + s * C::kTileBytes);
            const uint32_t dS = tmem + ((t & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss(dS, sdesc_sw128(sQ + koff, 16, 1024), sdesc_sw128(sK + koff, 16, 1024), idS,
                       kk > 0);
            }
            mma_commit(&bars->s_full[t & 1]);
            return true;
        };
        if (ok) ok = issue_S(0);
        for (int t = 0; ok && t < num_kv; ++t) {
            if (t + 1 < num_kv && !issue_S(t + 1)) { ok = false; break; }
            if (!mbar_wait(&bars->p_full[t & 1], (t >> 1) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int s = t % C::kStages;
            const uint32_t sV = smem_addr(smem + C::kOffV + s * C::kTileBytes);
            const uint32_t aP = tmem + ((t & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
                mma_ts(tmem + C::kColO, aP + kk * 8,
                       sdesc_sw128(sV + kk * 2048, C::kPanelBytes, 1024), idO, (t > 0 || kk > 0));
            mma_commit(&bars->kv_empty[s]);
            mma_commit(&bars->o_done);
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        // Drain: all MMAs issued here complete before TMEM is released.
        mma_commit(&bars->mma_drain);
        (void)mbar_wait_timed(&bars->mma_drain, 0, budget_ns);
    } else if (!aborted_early && warp >= 4) {
        // ------------------------------------------------ softmax warpgroup
        const int r = threadIdx.x - 128;               // query row in the tile == TMEM lane
        const uint32_t lane_sel = uint32_t((warp & 3) * 32) << 16;
        const int row = q0 + r;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < num_kv; ++t) {
            if (!mbar_wait_warp(&bars->s_full[t & 1], (t >> 1) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tmem + lane_sel + ((t & 1) ? C::kColS1 : C::kColS0);
            float sv[kBN];
#pragma unroll
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t rr[32];
                tmem_ld32(tS + c * 32, rr);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(rr[e]) * scale_log2;
            }
            const int k0 = t * kBN;
            const bool need_mask = (k0 + kBN > m) || (causal && k0 + kBN - 1 > q0);
            if (need_mask) {
#pragma unroll
                for (int e = 0; e < kBN; ++e) {
                    const int key = k0 + e;
                    if (key >= m || (causal && key > row)) sv[e] = -INFINITY;
                }
            }
            float tmax = -INFINITY;
#pragma unroll
            for (int e = 0; e < kBN; ++e) tmax = fmaxf(tmax, sv[e]);
            const float m_new = fmaxf(m_run, tmax);
            const bool want = m_new > m_run + kRescaleThreshold;   // true on the first tile
            const bool warp_rescale = __any_sync(0xffffffffu, want && t > 0);
            float alpha = 1.f;
            if (want) {
                alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
                m_run = m_new;
                l_run *= alpha;
            }
            if (warp_rescale) {
                // O must hold P_{t-1} V_{t-1} before it is rescaled.
                if (!mbar_wait_warp(&bars->o_done, (t - 1) & 1, abort_flag, budget_ns)) ok = false;
                tc_fence_after();
                const uint32_t tO = tmem + lane_sel + C::kColO;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(tO + c * 32, rr);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
                    tmem_st32(tO + c * 32, rr);
                }
            }
            const float msub = (m_run == -INFINITY) ? 0.f : m_run;
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = ex2(sv[c * 32 + 2 * e] - msub);
                    const float p1 = ex2(sv[c * 32 + 2 * e + 1] - msub);
                    lsum += p0 + p1;
                    pk[e] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tS + c * 16, pk);     // P over S columns already read
            }
            l_run += lsum;
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars->p_full[t & 1]);
            if (!ok) break;
        }
        if (ok && num_kv > 0 &&
            !mbar_wait_warp(&bars->o_done, (num_kv - 1) & 1, abort_flag, budget_ns))
            ok = false;
        if (ok) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            const uint32_t tO = tmem + lane_sel + C::kColO;
            __nv_bfloat16* orow = O + (size_t(bh) * n + row) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t rr[32];
                tmem_ld32(tO + c * 32, rr);
                tmem_ld_wait();
                if (row < n) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(rr[8 * v + 0]) * inv, __uint_as_float(rr[8 * v + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(rr[8 * v + 2]) * inv, __uint_as_float(rr[8 * v + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(rr[8 * v + 4]) * inv, __uint_as_float(rr[8 * v + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(rr[8 * v + 6]) * inv, __uint_as_float(rr[8 * v + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + 8 * v) = w;
                    }
                }
            }
            if (row < n) LSE[size_t(bh) * n + row] = (m_run + log2f(l_run)) * kLn2;
        } else {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fwdtc
}  // namespace attn
