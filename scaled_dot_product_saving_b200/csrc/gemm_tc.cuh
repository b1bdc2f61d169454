// gemm_tc.cuh -- tensor-core GEMM for the projection gradients of
// self-attention ("Lesson 4 - The Backward Pass for Attention", section
// "Step 4: Back to the Parameters and Input"; "Attention backward",
// Problem 7): dW = X^T dQ (summed over the batch) and dX = dQ Wq^T + ...
//
//   D[m][n] = sum_k A(m, k) B(k, n),   bf16 operands, fp32 accumulation in
//   TMEM, bf16 result.
//
// A is read through a tensor map (3-D, last extent 1) either K-major (stored [M][K]) or
// MN-major (stored [K][M], i.e. A^T row-major); B likewise (K-major: stored
// [N][K]; MN-major: stored [K][N]). One CTA computes a 128 x 256 tile of D
// over K in blocks of 64, with a 4-stage TMA ring: warp 0 loads, warp 1
// allocates TMEM and issues the MMAs (4 per K block, M = 128, N = 256,
// K = 16 each), warps 2-5 read the accumulator out of TMEM (one row per
// thread) and store it. Tiles and K blocks that run past the matrix edges
// are zero-filled by the TMA; the stores are clipped.
#pragma once

#include "sm100.cuh"

namespace attn {
namespace gemmtc {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kGroupM = 8;     // row tiles per rasterisation group
constexpr int kThreads = 192;
constexpr int kABytes = kBM * kBK * 2;          // 16 KB
constexpr int kBBytes = kBN * kBK * 2;          // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kSmemBytes = kOffBar + 256;
constexpr uint32_t kTmemCols = 256;

struct Bars {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;
    uint64_t mma_drain;
    uint32_t tmem_base;
    int abort;
};

template <bool A_KMAJOR, bool B_KMAJOR>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            __nv_bfloat16* __restrict__ D, int M, int N, int K, int ldd,
            unsigned long long budget_ns) {
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    volatile int* abort_flag = &bars->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Tile order: groups of kGroupM row tiles, column tiles across each group,
    // so the CTAs in flight share their A row panels and B column panels in L2.
    const int mt = (M + kBM - 1) / kBM, nt = (N + kBN - 1) / kBN;
    const int b = int(blockIdx.x);
    const int group = b / (kGroupM * nt);
    const int gm = min(kGroupM, mt - group * kGroupM);
    const int within = b - group * kGroupM * nt;
    const int m0 = (group * kGroupM + within % gm) * kBM, n0 = (within / gm) * kBN;
    const int num_kb = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        const bool misaligned = (smem_addr(smem) & 1023u) != 0;
        if (misaligned) record_device_error(kErrTimeout);
        bars->abort = (misaligned || *reinterpret_cast<volatile unsigned int*>(&g_device_error) != 0) ? 1 : 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->mma_drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const bool aborted_early = bars->abort != 0;

    if (!aborted_early && warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        prefetch_tensor_map(&tmA);
        prefetch_tensor_map(&tmB);
        int issued = 0;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % kStages;
            if (kb >= kStages &&
                !mbar_wait(&bars->empty[s], (kb / kStages - 1) & 1, abort_flag, budget_ns)) {
                record_device_error(kErrTimeout);
                *abort_flag = 1;
                break;
            }
            uint8_t* sa = smem + s * kStageBytes;
            uint8_t* sb = sa + kABytes;
            const int k0 = kb * kBK;
            mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
            // A: K-major, one 128-row x 128-byte box; MN-major, two 64-row
            // (K) x 64-column (M) panels.
            if (A_KMAJOR) {
                tma_load_3d(sa, &tmA, &bars->full[s], k0, m0, 0);
            } else {
                tma_load_3d(sa, &tmA, &bars->full[s], m0, k0, 0);
                tma_load_3d(sa + 8192, &tmA, &bars->full[s], m0 + 64, k0, 0);
            }
            // B: K-major, one 256-row box; MN-major, four 64 x 64 panels.
            if (B_KMAJOR) {
                tma_load_3d(sb, &tmB, &bars->full[s], k0, n0, 0);
            } else {
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    tma_load_3d(sb + p * 8192, &tmB, &bars->full[s], n0 + 64 * p, k0, 0);
            }
            ++issued;
        }
        for (int kb = (issued > kStages ? issued - kStages : 0); kb < issued; ++kb)
            (void)mbar_wait_timed(&bars->full[kb % kStages], (kb / kStages) & 1, budget_ns);
    } else if (!aborted_early && warp == 1) {
        // ------------------------------------------------ MMA issuer
        // The whole warp walks the loop (waits are warp-wide) and one elected
        // lane issues the MMAs and commits.
        const uint32_t leader = elect_leader();
        constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, A_KMAJOR ? 0 : 1, B_KMAJOR ? 0 : 1);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait_warp(&bars->full[s], (kb / kStages) & 1, abort_flag, budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sa = smem_addr(smem + s * kStageBytes);
            const uint32_t sb = sa + kABytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                // K-major: a K step is 32 bytes along the 128-byte row;
                // MN-major: 16 rows of 128 bytes, 64-wide panels 8 KB apart.
                const uint64_t da = A_KMAJOR ? sdesc_at(sa, kk * 32, 16, 1024)
                                             : sdesc_at(sa, kk * 2048, 8192, 1024);
                const uint64_t db = B_KMAJOR ? sdesc_at(sb, kk * 32, 16, 1024)
                                             : sdesc_at(sb, kk * 2048, 8192, 1024);
                mma_ss_w(tmem, da, db, idesc, (kb > 0 || kk > 0) ? 1u : 0u, leader);
            }
            mma_commit_w(&bars->empty[s], leader);
        }
        if (ok) mma_commit_w(&bars->acc_full, leader);
        else {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
        mma_commit_w(&bars->mma_drain, leader);
        (void)mbar_wait_timed(&bars->mma_drain, 0, budget_ns);
    } else if (!aborted_early && warp >= 2) {
        // ------------------------------------------------ epilogue
        // Warp w reads TMEM lanes 32 (w % 4) .. +31: row m0 + that lane.
        const int q = warp & 3;
        const int row = m0 + q * 32 + lane;
        const uint32_t tl = tmem + (uint32_t(q * 32) << 16);
        if (mbar_wait_warp(&bars->acc_full, 0, abort_flag, budget_ns)) {
            tc_fence_after();
            __nv_bfloat16* drow = D + size_t(row) * ldd;
            const bool vec_ok = (ldd % 8) == 0;
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tl + 32 * c, r);
                tmem_ld_wait(r);
                if (row < M) {
                    const int nc = n0 + 32 * c;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int n = nc + 8 * v;
                        if (vec_ok && n + 8 <= N) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                            w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                            w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                            w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                            *reinterpret_cast<uint4*>(drow + n) = w;
                        } else {
                            for (int e = 0; e < 8; ++e)
                                if (n + e < N) drow[n + e] = __float2bfloat16_rn(__uint_as_float(r[8 * v + e]));
                        }
                    }
                }
            }
        } else {
            record_device_error(kErrTimeout);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace gemmtc
}  // namespace attn
