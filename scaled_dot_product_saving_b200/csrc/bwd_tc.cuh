// bwd_tc.cuh -- tensor-core backward for bf16, d == dv in {64, 128}.
//
// Key-tile major. One CTA owns 128 keys (K_j, V_j resident in shared memory)
// of one (batch, head) and walks the 128-row query tiles i that can see them
// (i >= j when causal). Per query tile, with keys as the MMA's M dimension:
//   S^T  = K_j Q_i^T                  tcgen05 (A = K_j, B = Q_i, both K-major)
//   dP^T = V_j dO_i^T                 tcgen05 (A = V_j, B = dO_i)
//   P^T  = 2^(S^T*scale*log2e - LSE_i*log2e), 0 where masked
//   dS^T = scale * P^T * (dP^T - D_i)            (128 threads, one key each)
//   dV_j += P^T dO_i                  tcgen05, A = P^T from TMEM (bf16 written
//                                     over its own S^T columns), B = dO_i MN-major
//   dK_j += dS^T Q_i                  tcgen05, A = dS^T from TMEM, B = Q_i MN-major
//   dQ_i += dS K_j                    tcgen05, A = dS from shared memory
//                                     (MN-major), B = K_j (MN-major); the fp32
//                                     result is reduce-added into the global dQ
//                                     accumulator by a second warpgroup.
// dV_j and dK_j stay in TMEM across all query tiles and are written once.
// Folding `scale` into dS makes dK and dQ come out already scaled.
//
// Where the pages stand: dV, dP, dS, dQ and dK are "Attention Backward Pass
// (dQ, dK, dV)", section "Backward", and "Attention backward", Problems 2-6;
// D = rowsum(dO * O) replaces rowsum(dP * P) per "Attention Backpropagation:
// Step by step derivation", section "Gradient of S"; masked dS entries are
// exact zeros ("Attention backward", Problem 8), so tiles wholly above the
// diagonal are skipped.
//
// Warp roles (384 threads): warp 0 = TMA producer, warp 1 = TMEM allocator and
// MMA issuer, warps 4-7 = P/dS warpgroup (TMEM lane = key), warps 8-11 = dQ
// warpgroup (TMEM lane = query row).
//
// TMEM (512 columns). d = 128: dV [0,128) dK [128,256) S^T [256,384)
// dP^T [384,512); P^T (bf16) goes to [256,320), dS^T to [384,448), and the two
// 64-column halves of dQ to [320,384) and [448,512) -- columns whose fp32
// contents have been consumed by then. d = 64: dV [0,64) dK [64,128)
// S^T [128,256) dP^T [256,384) dQ [384,448).
#pragma once

#include "sm100.cuh"

namespace attn {
namespace bwdtc {

constexpr int kBN = 128;      // keys per CTA
constexpr int kBM = 128;      // queries per tile
constexpr int kThreads = 384;

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
    static constexpr int kOffdS = kOffdO + kStages * kTileBytes;   // 128 keys x 128 queries
    static constexpr int kOffLse = kOffdS + 128 * 128 * 2;
    static constexpr int kOffDd = kOffLse + kStages * kBM * 4;
    static constexpr int kOffBar = kOffDd + kStages * kBM * 4;
    static constexpr int kSmemBytes = kOffBar + 256;
    static constexpr bool kAlias = (D == 128);
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColdV = 0;
    static constexpr uint32_t kColdK = D;
    static constexpr uint32_t kColS = 2 * D;
    static constexpr uint32_t kColdP = 2 * D + 128;
    static constexpr uint32_t kColP = kColS;          // bf16 P^T over S^T
    static constexpr uint32_t kColdS = kColdP;        // bf16 dS^T over dP^T
    static constexpr uint32_t kColdQ0 = kAlias ? kColS + 64 : 2 * D + 256;
    static constexpr uint32_t kColdQ1 = kAlias ? kColdP + 64 : kColdQ0 + 64;
};

struct Bars {
    uint64_t kv_full;
    uint64_t q_full[4];
    uint64_t q_empty[4];
    uint64_t s_full;
    uint64_t ds_full;
    uint64_t dq_full;
    uint64_t dq_free;
    uint64_t acc_done;
    uint64_t mma_drain;
    uint32_t tmem_base;
    int abort;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
           const float* __restrict__ lse2, const float* __restrict__ Dd, int n_pad,
           float* __restrict__ dQacc, __nv_bfloat16* __restrict__ dK,
           __nv_bfloat16* __restrict__ dV, int n, int m, int BH, int causal, float scale,
           float scale_log2, unsigned long long budget_ns) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt = int(blockIdx.x / BH);      // key tile; low tiles (most work if causal) first
    const int bh = int(blockIdx.x % BH);
    const int k0 = kt * kBN;
    const int num_qt = (n + kBM - 1) / kBM;
    const int first_qt = causal ? kt : 0;
    const int T = num_qt - first_qt;          // query tiles this CTA visits (>= 1)

    if (threadIdx.x == 0) {
        // The swizzled tiles need a 1024-byte aligned base. A CTA that starts
        // after another one gave up a wait does no work at all.
        const bool misaligned = (smem_addr(smem) & 1023u) != 0;
        if (misaligned) record_device_error(kErrTimeout);
        bars->abort = (misaligned || *reinterpret_cast<volatile unsigned int*>(&g_device_error) != 0) ? 1 : 0;
        mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->ds_full, 128);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_free, 128);
        mbar_init(&bars->acc_done, 1);
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
    const bool aborted_early = bars->abort != 0 || T <= 0;

    if (!aborted_early && warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        prefetch_tensor_map(&tmQ);
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        prefetch_tensor_map(&tmdO);
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p) {
            tma_load_3d(smem + C::kOffK + p * C::kPanelBytes, &tmK, &bars->kv_full, p * 64, k0, bh);
            tma_load_3d(smem + C::kOffV + p * C::kPanelBytes, &tmV, &bars->kv_full, p * 64, k0, bh);
        }
        int issued = 0;
        for (int t = 0; t < T; ++t) {
            const int s = t % C::kStages, k = t / C::kStages;
            const int q0 = (first_qt + t) * kBM;
            if (t >= C::kStages &&
                !mbar_wait(&bars->q_empty[s], (k - 1) & 1, abort_flag, budget_ns)) {
                record_device_error(kErrTimeout);
                *abort_flag = 1;
                break;
            }
            mbar_arrive_expect_tx(&bars->q_full[s], 2 * C::kTileBytes + 2 * kBM * 4);
            for (int p = 0; p < C::kPanels; ++p) {
                tma_load_3d(smem + C::kOffQ + s * C::kTileBytes + p * C::kPanelBytes, &tmQ,
                            &bars->q_full[s], p * 64, q0, bh);
                tma_load_3d(smem + C::kOffdO + s * C::kTileBytes + p * C::kPanelBytes, &tmdO,
                            &bars->q_full[s], p * 64, q0, bh);
            }
            bulk_load(smem + C::kOffLse + s * kBM * 4, lse2 + size_t(bh) * n_pad + q0, kBM * 4,
                      &bars->q_full[s]);
            bulk_load(smem + C::kOffDd + s * kBM * 4, Dd + size_t(bh) * n_pad + q0, kBM * 4,
                      &bars->q_full[s]);
            ++issued;
        }
        (void)mbar_wait_timed(&bars->kv_full, 0, budget_ns);
        for (int t = (issued > C::kStages ? issued - C::kStages : 0); t < issued; ++t)
            (void)mbar_wait_timed(&bars->q_full[t % C::kStages], (t / C::kStages) & 1, budget_ns);
    } else if (!aborted_early && warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idSP = idesc_bf16_f32(kBN, kBM, 0, 0);   // S^T, dP^T
        constexpr uint32_t idKV = idesc_bf16_f32(kBN, D, 0, 1);     // dV, dK
        constexpr uint32_t idQ = idesc_bf16_f32(kBM, 64, 1, 1);     // dQ, one 64-wide half
        const uint32_t sK = smem_addr(smem + C::kOffK);
        const uint32_t sV = smem_addr(smem + C::kOffV);
        const uint32_t sdS = smem_addr(smem + C::kOffdS);
        bool ok = mbar_wait(&bars->kv_full, 0, abort_flag, budget_ns);
        for (int t = 0; ok && t < T; ++t) {
            const int s = t % C::kStages;
            const uint32_t sQ = smem_addr(smem + C::kOffQ + s * C::kTileBytes);
            const uint32_t sdO = smem_addr(smem + C::kOffdO + s * C::kTileBytes);
            if (!mbar_wait(&bars->q_full[s], (t / C::kStages) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            if (C::kAlias && t > 0 &&
                !mbar_wait(&bars->dq_free, (t - 1) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss(tmem + C::kColS, sdesc_sw128(sK + koff, 16, 1024),
                       sdesc_sw128(sQ + koff, 16, 1024), idSP, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                mma_ss(tmem + C::kColdP, sdesc_sw128(sV + koff, 16, 1024),
                       sdesc_sw128(sdO + koff, 16, 1024), idSP, kk > 0);
            }
            mma_commit(&bars->s_full);
            if (!mbar_wait(&bars->ds_full, t & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kBM / 16; ++kk)
                mma_ts(tmem + C::kColdV, tmem + C::kColP + kk * 8,
                       sdesc_sw128(sdO + kk * 2048, C::kPanelBytes, 1024), idKV, (t > 0 || kk > 0));
#pragma unroll
            for (int kk = 0; kk < kBM / 16; ++kk)
                mma_ts(tmem + C::kColdK, tmem + C::kColdS + kk * 8,
                       sdesc_sw128(sQ + kk * 2048, C::kPanelBytes, 1024), idKV, (t > 0 || kk > 0));
            mma_commit(&bars->q_empty[s]);
            if (t == T - 1) mma_commit(&bars->acc_done);
            if (!C::kAlias && t > 0 &&
                !mbar_wait(&bars->dq_free, (t - 1) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int h = 0; h < C::kPanels; ++h) {
                const uint32_t dq = tmem + (h == 0 ? C::kColdQ0 : C::kColdQ1);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ss(dq, sdesc_sw128(sdS + kk * 2048, C::kPanelBytes, 1024),
                           sdesc_sw128(sK + h * C::kPanelBytes + kk * 2048, C::kPanelBytes, 1024),
                           idQ, kk > 0);
            }
            mma_commit(&bars->dq_full);
        }
        if (!ok) {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        mma_commit(&bars->mma_drain);
        (void)mbar_wait_timed(&bars->mma_drain, 0, budget_ns);
    } else if (!aborted_early && warp >= 4 && warp < 8) {
        // ------------------------------------------------ P / dS warpgroup
        const int r = threadIdx.x - 128;                 // key row in the tile == TMEM lane
        const uint32_t lane_sel = uint32_t((warp & 3) * 32) << 16;
        const int j = k0 + r;
        const bool key_ok = j < m;
        uint8_t* sdS = smem + C::kOffdS;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int s = t % C::kStages;
            const int q0 = (first_qt + t) * kBM;
            if (!mbar_wait_warp(&bars->q_full[s], (t / C::kStages) & 1, abort_flag, budget_ns) ||
                !mbar_wait_warp(&bars->s_full, t & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float* lse_s = reinterpret_cast<const float*>(smem + C::kOffLse + s * kBM * 4);
            const float* dd_s = reinterpret_cast<const float*>(smem + C::kOffDd + s * kBM * 4);
            const bool diag = causal && (q0 == k0);
#pragma unroll
            for (int c = 0; c < kBM / 32; ++c) {
                uint32_t sr[32], pr[32];
                tmem_ld32(tmem + lane_sel + C::kColS + c * 32, sr);
                tmem_ld32(tmem + lane_sel + C::kColdP + c * 32, pr);
                tmem_ld_wait();
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float pp[2], dd[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int qi = c * 32 + 2 * e + h;
                        float p = ex2(fmaf(__uint_as_float(sr[2 * e + h]), scale_log2, -lse_s[qi]));
                        if (!key_ok || (diag && qi < r)) p = 0.f;
                        pp[h] = p;
                        dd[h] = p * (__uint_as_float(pr[2 * e + h]) - dd_s[qi]) * scale;
                    }
                    pk[e] = pack_bf16x2(pp[0], pp[1]);
                    dk[e] = pack_bf16x2(dd[0], dd[1]);
                }
                tmem_st16(tmem + lane_sel + C::kColP + c * 16, pk);
                tmem_st16(tmem + lane_sel + C::kColdS + c * 16, dk);
                // dS (queries contiguous, 128B-swizzled) for the dQ MMA's A operand.
                uint8_t* rowp = sdS + (c >> 1) * C::kPanelBytes + r * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = ((c & 1) * 4 + q) ^ (r & 7);
                    *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                        make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_full);
        }
        if (ok && !mbar_wait_warp(&bars->acc_done, 0, abort_flag, budget_ns)) ok = false;
        if (ok) {
            tc_fence_after();
            __nv_bfloat16* vrow = dV + (size_t(bh) * m + j) * D;
            __nv_bfloat16* krow = dK + (size_t(bh) * m + j) * D;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col = which == 0 ? C::kColdV : C::kColdK;
                __nv_bfloat16* dst = which == 0 ? vrow : krow;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(tmem + lane_sel + col + c * 32, rr);
                    tmem_ld_wait();
                    if (key_ok) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(rr[8 * v + 0]), __uint_as_float(rr[8 * v + 1]));
                            w.y = pack_bf16x2(__uint_as_float(rr[8 * v + 2]), __uint_as_float(rr[8 * v + 3]));
                            w.z = pack_bf16x2(__uint_as_float(rr[8 * v + 4]), __uint_as_float(rr[8 * v + 5]));
                            w.w = pack_bf16x2(__uint_as_float(rr[8 * v + 6]), __uint_as_float(rr[8 * v + 7]));
                            *reinterpret_cast<uint4*>(dst + c * 32 + 8 * v) = w;
                        }
                    }
                }
            }
        } else {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
    } else if (!aborted_early && warp >= 8) {
        // ------------------------------------------------ dQ warpgroup
        const int r = threadIdx.x - 256;                 // query row in the tile == TMEM lane
        const uint32_t lane_sel = uint32_t((warp & 3) * 32) << 16;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int i = (first_qt + t) * kBM + r;
            if (!mbar_wait_warp(&bars->dq_full, t & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t v[D];
#pragma unroll
            for (int h = 0; h < C::kPanels; ++h) {
                const uint32_t col = h == 0 ? C::kColdQ0 : C::kColdQ1;
                tmem_ld32(tmem + lane_sel + col, *reinterpret_cast<uint32_t(*)[32]>(v + 64 * h));
                tmem_ld32(tmem + lane_sel + col + 32,
                          *reinterpret_cast<uint32_t(*)[32]>(v + 64 * h + 32));
            }
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&bars->dq_free);
            if (i < n) {
                float* dst = dQacc + (size_t(bh) * n + i) * D;
#pragma unroll
                for (int c = 0; c < D; c += 4)
                    red_add_v4(dst + c, __uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                               __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
            }
        }
        if (!ok) {
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

}  // namespace bwdtc
}  // namespace attn
