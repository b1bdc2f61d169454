// f32x_tc.cuh -- fp32 attention forward and backward on the tensor cores, by
// splitting every fp32 operand into three bf16 pieces.
//
// The arithmetic is that of "Attention Backward Pass (dQ, dK, dV) -
// Transformer Architecture", sections "Forward" and "Backward", as in the
// bf16 kernels: S = scale Q K^T, P = softmax(S) (causal: key j > query i
// masked), O = P V, and with D = rowsum(dO * O) ("Attention Backpropagation:
// Step by step derivation", section "Gradient of S"): dV = P^T dO,
// dS = P * (dO V^T - D), dQ = scale dS K, dK = scale dS^T Q.
//
// Precision. A value x in fp32 is written exactly as x0 + x1 + x2 with
//   x0 = bf16(x) (rounded to nearest),  x1 = x - x0 truncated to bf16,
//   x2 = x - x0 - x1 (at most 8 significant bits, so a bf16 value)
// (both subtractions are exact in fp32); |x1| <= 2^-8 |x| and |x2| < 2^-16
// |x|. A product a b is the sum of the six piece products a_i b_j with
// i + j <= 2; the three left out are below about 2^-23 |a b| together. Each piece product is one bf16 tcgen05 MMA accumulating in fp32
// in TMEM, so one fp32 contraction costs six bf16 MMAs -- the tensor time of
// three tf32 MMAs (tf32 runs at half the bf16 rate), with operands rounded to
// 24 significant bits instead of the 22 of a tf32 hi/lo pair, and with the
// operand layouts of the bf16 kernels.
//
// Shapes. Operands are zero-padded to 64 columns, so d, dv <= 64 (multiples
// of 4 for 16-byte loads). Every MMA is M = 128, N = 64, K = 16: the 128 rows
// a CTA owns sit one per TMEM lane, the streamed tiles have 64 rows. Pieces
// of a tile are stored one after another, each in the 128-byte swizzled
// layout the MMA descriptors read (rows of 64 bf16).
//
// Kernels (256 threads; thread t owns row t % 128 and the column half t / 128
// of it; one elected thread issues the MMAs, all threads load, split and run
// the elementwise steps):
//   fwd_kernel     a 128-query tile, 64-key tiles: S (SS), online softmax in
//                  registers (the halves trade row maxima through shared
//                  memory), P split into TMEM, P V (TS) added into O in
//                  registers with the running rescale.
//   bwd_kernel     two passes in one launch:
//     kv_pass      a 128-key tile, 64-query tiles: S^T, dP^T (SS), P^T and
//                  dS^T split into TMEM, dV += P^T dO and dK += dS^T Q (TS).
//     dq_pass      a 128-query tile, 64-key tiles: S, dP (SS), dS split into
//                  TMEM, dQ += dS K (TS). dQ is written once, no atomics.
// The backward is two passes that each recompute S and dP, so that neither
// needs a transposed copy of dS in shared memory (three pieces of a 128 x 128
// tile would not fit beside the operands). Streamed tiles are double
// buffered. In both passes the next tile's S/dP MMAs are issued before this
// tile's dV/dK (dQ) MMAs, so the elementwise step of the next tile runs
// under them; its pieces go to TMEM once they are done, when the buffer of
// the tile before is also reloaded.
//
// The backward takes D multiplied by the scale and the LSE in base 2, from
// the preprocess kernel (padded to whole 128-row tiles: LSE = +inf and D = 0
// in the padding, so padded query rows get P = 0).
#pragma once

#include "sm100.cuh"
#include "padmask.cuh"

namespace attn {
namespace f32x {

constexpr int kBig = 128;                       // rows a CTA owns (= threads = TMEM lanes)
constexpr int kSmall = 64;                      // rows of a streamed tile
constexpr int kWidth = 64;                      // padded operand width
constexpr int kBigPiece = kBig * 128;           // one bf16 piece of a 128 x 64 tile
constexpr int kSmallPiece = kSmall * 128;       // one bf16 piece of a 64 x 64 tile
constexpr int kBigTile = 3 * kBigPiece;         // 48 KB
constexpr int kSmallTile = 3 * kSmallPiece;     // 24 KB
constexpr float kLn2 = 0.6931471805599453f;

// The six piece pairs (a, b) with a + b <= 2, smallest products first.
__host__ __device__ constexpr int pair_a(int p) { return p == 0 ? 2 : p == 1 ? 1 : p == 2 ? 0 : p == 3 ? 1 : 0; }
__host__ __device__ constexpr int pair_b(int p) { return p == 0 ? 0 : p == 1 ? 1 : p == 2 ? 2 : p == 3 ? 0 : p == 4 ? 1 : 0; }

struct Bars {
    uint64_t bar_a;       // first MMA group of a step has completed
    uint64_t bar_b;       // second MMA group of a step has completed
    uint64_t drain;       // every MMA of the CTA has completed (teardown)
    uint32_t tmem_base;
};

// ------------------------------------------------------------ splitting
__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 h) {
    return *reinterpret_cast<uint32_t*>(&h);
}

// Two fp32 values (x: lower element) into their three bf16 pieces, packed
// two to a word: x0 = bf16(x) rounded to nearest, x1 = x - x0 truncated to
// bf16 (its upper 16 bits), x2 = x - x0 - x1. Both subtractions are exact,
// and x2 has at most 8 significant bits, so x0 + x1 + x2 = x exactly with one
// float-to-bf16 conversion per pair (the conversion pipe is the narrow one).
__device__ __forceinline__ void split2(float x, float y, uint32_t& w0, uint32_t& w1, uint32_t& w2) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(x, y);
    const float2 f0 = __bfloat1622float2(h0);
    const float rx = __fsub_rn(x, f0.x), ry = __fsub_rn(y, f0.y);
    const uint32_t ux = __float_as_uint(rx) & 0xffff0000u, uy = __float_as_uint(ry) & 0xffff0000u;
    const float sx = __fsub_rn(rx, __uint_as_float(ux)), sy = __fsub_rn(ry, __uint_as_float(uy));
    w0 = bf2_bits(h0);
    w1 = __byte_perm(ux, uy, 0x7632);
    w2 = __byte_perm(__float_as_uint(sx), __float_as_uint(sy), 0x7632);
}

// Rows [row0, row0 + R) of a row-major [rows_valid, width] fp32 matrix into
// the three pieces at `dst` (R * 128 bytes apart), 128-byte swizzled rows of
// 64 bf16. Rows at or past rows_valid and columns at or past width are zero.
// width % 4 == 0; the matrix starts 16-byte aligned.
template <int R, int NT>
__device__ __forceinline__ void load_split(const float* __restrict__ src, int row0, int rows_valid,
                                           int width, uint8_t* dst, int tid) {
#pragma unroll 2
    for (int k = tid; k < R * 8; k += NT) {
        const int r = k >> 3, c = k & 7;
        const int grow = row0 + r, col = 8 * c;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (grow < rows_valid && col < width) {
            const float4* p = reinterpret_cast<const float4*>(src + size_t(grow) * width + col);
            a = __ldg(p);
            if (col + 8 <= width) b = __ldg(p + 1);
        }
        uint4 p0, p1, p2;
        split2(a.x, a.y, p0.x, p1.x, p2.x);
        split2(a.z, a.w, p0.y, p1.y, p2.y);
        split2(b.x, b.y, p0.z, p1.z, p2.z);
        split2(b.z, b.w, p0.w, p1.w, p2.w);
        const int off = r * 128 + ((c ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst + off) = p0;
        *reinterpret_cast<uint4*>(dst + R * 128 + off) = p1;
        *reinterpret_cast<uint4*>(dst + 2 * R * 128 + off) = p2;
    }
}

// load_split of two matrices with the same rows (K and V, or Q and dO): all
// of a thread's loads are issued before any is split, so that the prologue
// of a CTA waits for memory once rather than once per matrix and chunk.
template <int R, int NT>
__device__ __forceinline__ void load_split2(const float* __restrict__ srcA, int widthA, uint8_t* dstA,
                                            const float* __restrict__ srcB, int widthB, uint8_t* dstB,
                                            int row0, int rows_valid, int tid) {
    static_assert((R * 8) % NT == 0, "whole chunks per thread");
    constexpr int kIters = R * 8 / NT;
    float4 a[2][kIters], b[2][kIters];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const float* src = m ? srcB : srcA;
        const int width = m ? widthB : widthA;
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            const int k = tid + it * NT;
            const int r = k >> 3, col = 8 * (k & 7);
            const int grow = row0 + r;
            a[m][it] = b[m][it] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (grow < rows_valid && col < width) {
                const float4* ptr = reinterpret_cast<const float4*>(src + size_t(grow) * width + col);
                a[m][it] = __ldg(ptr);
                if (col + 8 <= width) b[m][it] = __ldg(ptr + 1);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        uint8_t* dst = m ? dstB : dstA;
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            const int k = tid + it * NT;
            const int r = k >> 3, c = k & 7;
            uint4 p0, p1, p2;
            split2(a[m][it].x, a[m][it].y, p0.x, p1.x, p2.x);
            split2(a[m][it].z, a[m][it].w, p0.y, p1.y, p2.y);
            split2(b[m][it].x, b[m][it].y, p0.z, p1.z, p2.z);
            split2(b[m][it].z, b[m][it].w, p0.w, p1.w, p2.w);
            const int off = r * 128 + ((c ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(dst + off) = p0;
            *reinterpret_cast<uint4*>(dst + R * 128 + off) = p1;
            *reinterpret_cast<uint4*>(dst + 2 * R * 128 + off) = p2;
        }
    }
}

// Asynchronous 16-byte global -> shared copies (zero-filled past src_bytes).
__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(sdst)),
                 "l"(gsrc), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// The fp32 rows that load_split would read, copied as they are into `stage`
// (32 bytes per 8-column chunk, in chunk order) without waiting. Each thread
// copies the chunks it will later split itself (split_staged), so neither
// step needs a barrier. The caller commits the copies as one group.
template <int R, int NT>
__device__ __forceinline__ void fetch(const float* __restrict__ src, int row0, int rows_valid,
                                      int width, uint8_t* stage, int tid) {
#pragma unroll 2
    for (int k = tid; k < R * 8; k += NT) {
        const int r = k >> 3, col = 8 * (k & 7);
        const int grow = row0 + r;
        const bool rv = grow < rows_valid;
        const float* g = rv ? src + size_t(grow) * width + col : src;
        const uint32_t n0 = (rv && col < width) ? 16u : 0u;
        const uint32_t n1 = (rv && col + 4 < width) ? 16u : 0u;
        cp_async16(stage + 32 * k, n0 ? g : src, n0);
        cp_async16(stage + 32 * k + 16, n1 ? g + 4 : src, n1);
    }
}

// Wait for this thread's copies, then split its chunks of `stage` into the
// three pieces at `dst` (layout as load_split).
template <int R, int NT>
__device__ __forceinline__ void split_staged(const uint8_t* stage, uint8_t* dst, int tid) {
    cp_async_wait_all();
#pragma unroll 2
    for (int k = tid; k < R * 8; k += NT) {
        const int r = k >> 3, c = k & 7;
        const float4 a = *reinterpret_cast<const float4*>(stage + 32 * k);
        const float4 b = *reinterpret_cast<const float4*>(stage + 32 * k + 16);
        uint4 p0, p1, p2;
        split2(a.x, a.y, p0.x, p1.x, p2.x);
        split2(a.z, a.w, p0.y, p1.y, p2.y);
        split2(b.x, b.y, p0.z, p1.z, p2.z);
        split2(b.z, b.w, p0.w, p1.w, p2.w);
        const int off = r * 128 + ((c ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst + off) = p0;
        *reinterpret_cast<uint4*>(dst + R * 128 + off) = p1;
        *reinterpret_cast<uint4*>(dst + 2 * R * 128 + off) = p2;
    }
}

// 32 values of this thread's row into the three pieces in TMEM: piece a of
// the 64-wide row at columns col + 32 a .. +31 (two bf16 per column), this
// half (h = 0, 1) at +16 h.
__device__ __forceinline__ void split_to_tmem(const float (&v)[32], uint32_t taddr) {
    uint32_t w0[16], w1[16], w2[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) split2(v[2 * e], v[2 * e + 1], w0[e], w1[e], w2[e]);
    tmem_st16(taddr, w0);
    tmem_st16(taddr + 32, w1);
    tmem_st16(taddr + 64, w2);
}

// ------------------------------------------------------------ MMA groups
// D (+)= sum over the six pairs of A_a B_b^T, K = 64. A: 128 rows, K-major,
// pieces a_stride bytes apart; B: 64 rows, K-major, pieces b_stride apart.
__device__ __forceinline__ void mma6_ss(uint32_t d, uint32_t sa, uint32_t a_stride, uint32_t sb,
                                        uint32_t b_stride, uint32_t idesc) {
#pragma unroll
    for (int p = 0; p < 6; ++p)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_ss(d, sdesc_at(sa + pair_a(p) * a_stride, kk * 32, 16, 1024),
                   sdesc_at(sb + pair_b(p) * b_stride, kk * 32, 16, 1024), idesc,
                   (p > 0 || kk > 0) ? 1u : 0u);
}

// D (+)= sum over the six pairs of A_a B_b, K = 64. A in TMEM (pieces 32
// columns apart, 8 columns per 16-deep step); B in shared memory, MN-major:
// 64 rows along K, 64 columns along N, pieces kSmallPiece apart.
__device__ __forceinline__ void mma6_ts(uint32_t d, uint32_t ta, uint32_t sb, uint32_t idesc,
                                        bool accumulate) {
#pragma unroll
    for (int p = 0; p < 6; ++p)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_ts(d, ta + 32 * pair_a(p) + 8 * kk,
                   sdesc_at(sb + pair_b(p) * kSmallPiece, kk * 2048, kSmallPiece, 1024), idesc,
                   (accumulate || p > 0 || kk > 0) ? 1u : 0u);
}

constexpr uint32_t kIdSS = idesc_bf16_f32(128, 64, 0, 0);   // both K-major
constexpr uint32_t kIdTS = idesc_bf16_f32(128, 64, 0, 1);   // B MN-major

// Common prologue / epilogue pieces.
__device__ __forceinline__ void init_bars(Bars* bars, uint32_t tmem_cols) {
    if (threadIdx.x == 0) {
        mbar_init(&bars->bar_a, 1);
        mbar_init(&bars->bar_b, 1);
        mbar_init(&bars->drain, 1);
        fence_mbar_init();
    }
    if ((threadIdx.x >> 5) == 0) {
        tmem_alloc(&bars->tmem_base, tmem_cols);
        tmem_relinquish();
    }
}

// Wait until every MMA issued by thread 0 has completed, then free TMEM.
__device__ __forceinline__ void teardown(Bars* bars, uint32_t tmem, uint32_t tmem_cols,
                                         uint64_t budget_ns) {
    cp_async_wait_all();
    if (threadIdx.x == 0) {
        mma_commit(&bars->drain);
        if (!mbar_wait_timed(&bars->drain, 0, budget_ns)) record_device_error(kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

// Columns [c0, c0 + 32) of a row, clipped to width (width, c0 multiples of 4).
__device__ __forceinline__ void store_half(float* row, int c0, const float (&v)[32], int width) {
#pragma unroll
    for (int c = 0; c < 32; c += 4)
        if (c0 + c < width)
            *reinterpret_cast<float4*>(row + c0 + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
}

// ================================================================ forward
// TMEM columns: S (64), P V of the current key tile (64), P pieces (96).
// Two warpgroups: thread t owns row t % 128 and the key (and value) column
// half t / 128 of it. The halves trade their row maxima through shared memory
// once per key tile, so both apply the same running maximum and rescale, and
// add up their row sums at the end.
constexpr int kFwdThreads = 256;
constexpr uint32_t kFwdColS = 0, kFwdColPV = 64, kFwdColP = 128, kFwdTmemCols = 256;
constexpr int kFwdOffQ = 0;
constexpr int kFwdOffK = kFwdOffQ + kBigTile;          // two buffers
constexpr int kFwdOffV = kFwdOffK + 2 * kSmallTile;    // two buffers
constexpr int kStageBytes = kSmall * 8 * 32;           // one fp32 64 x 64 tile in flight
constexpr int kFwdOffStage = kFwdOffV + 2 * kSmallTile; // K, V of tile t + 2
constexpr int kFwdOffX = kFwdOffStage + 2 * kStageBytes; // [2 halves][128 rows] floats
constexpr int kFwdOffBar = kFwdOffX + 2 * kBig * 4;
constexpr int kFwdSmemBytes = kFwdOffBar + 128;

// Grid: one CTA per (128-query tile, head), heads fastest; causal grids start
// with the last query tiles (the most key tiles).
__global__ void __launch_bounds__(kFwdThreads, 1)
fwd_kernel(const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
           float* __restrict__ O, float* __restrict__ LSE, int n, int m, int d, int dv, int BH,
           int causal, float scale_log2, const int* __restrict__ key_len, int H,
           unsigned long long budget_ns) {
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + kFwdOffBar);
    float* xch = reinterpret_cast<float*>(smem + kFwdOffX);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane128 = tid & 127, half = tid >> 7;
    const int num_qt = (n + kBig - 1) / kBig;
    const int bh = int(blockIdx.x % unsigned(BH));
    const int rank = int(blockIdx.x / unsigned(BH));
    const int qt = causal ? num_qt - 1 - rank : rank;
    const int q0 = qt * kBig, row = q0 + lane128;
    const float* Qh = Q + size_t(bh) * n * d;
    const float* Kh = K + size_t(bh) * m * d;
    const float* Vh = V + size_t(bh) * m * dv;
    const int mk = keys_valid(key_len, bh, H, m);        // keys past mk: padding
    const int nkt = (mk + kSmall - 1) / kSmall;
    const int T = causal ? min(nkt, (q0 + kBig - 1) / kSmall + 1) : nkt;

    uint8_t* stK = smem + kFwdOffStage;
    uint8_t* stV = stK + kStageBytes;
    auto fetch_kv = [&](int t) {
        fetch<kSmall, kFwdThreads>(Kh, t * kSmall, m, d, stK, tid);
        fetch<kSmall, kFwdThreads>(Vh, t * kSmall, m, dv, stV, tid);
        cp_async_commit();
    };

    init_bars(bars, kFwdTmemCols);
    const bool aligned = (smem_addr(smem) & 1023u) == 0;
    if (aligned) {
        // Key tiles 0 and 1 are split in place; tile 2 is in flight meanwhile.
        if (T > 2) fetch_kv(2);
        load_split<kBig, kFwdThreads>(Qh, q0, n, d, smem + kFwdOffQ, tid);
        load_split2<kSmall, kFwdThreads>(Kh, d, smem + kFwdOffK, Vh, dv, smem + kFwdOffV, 0, m, tid);
        if (T > 1) {
            load_split2<kSmall, kFwdThreads>(Kh, d, smem + kFwdOffK + kSmallTile, Vh, dv,
                                             smem + kFwdOffV + kSmallTile, kSmall, m, tid);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tq = tmem + (uint32_t((warp & 3) * 32) << 16);   // this warp's lanes
    const uint32_t tl = tq + 32 * half;                             // ... and column half
    const uint32_t sQ = smem_addr(smem + kFwdOffQ);
    const uint32_t sK = smem_addr(smem + kFwdOffK), sV = smem_addr(smem + kFwdOffV);
    const int never = 0;

    bool ok = aligned;
    if (!aligned && tid == 0) record_device_error(kErrTimeout);
    if (ok && tid == 0) {
        mma6_ss(tmem + kFwdColS, sQ, kBigPiece, sK, kSmallPiece, kIdSS);
        mma_commit(&bars->bar_a);
    }
    float o[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] = 0.f;
    float mrow = -INFINITY, lrow = 0.f;                  // lrow: this half's share of the sum

    for (int j = 0; ok && j < T; ++j) {
        const int buf = j & 1;
        const int kb = j * kSmall + 32 * half;            // first key of this half
        float s[32];
        float mx = -INFINITY;
        const bool got = mbar_wait_warp(&bars->bar_a, j & 1, &never, budget_ns);
        if (got) {
            tc_fence_after();
            uint32_t sr[32];
            tmem_ld32(tl + kFwdColS, sr);
            tmem_ld_wait(sr);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const int key = kb + c;
                float x = __uint_as_float(sr[c]) * scale_log2;
                if (key >= mk || (causal && key > row)) x = -INFINITY;
                s[c] = x;
                mx = fmaxf(mx, x);
            }
        }
        xch[half * kBig + lane128] = mx;
        if (__syncthreads_or(!got)) {
            ok = false;
            break;
        }
        // Both halves see the same two maxima, so mrow, base and alpha agree.
        const float mnew = fmaxf(mrow, fmaxf(mx, xch[(half ^ 1) * kBig + lane128]));
        const float base = (mnew == -INFINITY) ? 0.f : mnew;
        const float alpha = (mrow == -INFINITY) ? 0.f : ex2(mrow - base);
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            s[c] = ex2(s[c] - base);
            lsum += s[c];
        }
        lrow = lrow * alpha + lsum;
        mrow = mnew;
        // this half's 32 keys are K elements 32 half .. +31: columns 16 half ..
        split_to_tmem(s, tq + kFwdColP + 16 * half);
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            mma6_ts(tmem + kFwdColPV, tmem + kFwdColP, sV + buf * kSmallTile, kIdTS, false);
            mma_commit(&bars->bar_b);
            if (j + 1 < T) {
                mma6_ss(tmem + kFwdColS, sQ, kBigPiece, sK + (buf ^ 1) * kSmallTile, kSmallPiece,
                        kIdSS);
                mma_commit(&bars->bar_a);
            }
        }
        const bool got2 = mbar_wait_warp(&bars->bar_b, j & 1, &never, budget_ns);
        if (got2) {
            tc_fence_after();
            uint32_t pv[32];
            tmem_ld32(tl + kFwdColPV, pv);
            tmem_ld_wait(pv);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = fmaf(o[c], alpha, __uint_as_float(pv[c]));
            // K_j (read by S_j) and V_j (read by P_j V_j) are free: split
            // tile j + 2 from the staging buffer into them, then start
            // fetching tile j + 3.
            if (j + 2 < T) {
                split_staged<kSmall, kFwdThreads>(stK, smem + kFwdOffK + buf * kSmallTile, tid);
                split_staged<kSmall, kFwdThreads>(stV, smem + kFwdOffV + buf * kSmallTile, tid);
                fence_proxy_async_smem();
                if (j + 3 < T) fetch_kv(j + 3);
            }
        }
        tc_fence_before();
        if (__syncthreads_or(!got2)) {
            ok = false;
            break;
        }
    }

    if (ok) {
        // The row sum is the two halves' shares added (in the same order in
        // both halves).
        xch[half * kBig + lane128] = lrow;
        __syncthreads();
        const float l = xch[lane128] + xch[kBig + lane128];
        if (row < n) {
            const float inv = 1.0f / l;
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= inv;
            store_half(O + (size_t(bh) * n + row) * dv, 32 * half, o, dv);
            if (half == 0) LSE[size_t(bh) * n + row] = (mrow + log2f(l)) * kLn2;
        }
    } else if (tid == 0) {
        record_device_error(kErrTimeout);
    }
    teardown(bars, tmem, kFwdTmemCols, budget_ns);
}

// ================================================================ backward
// Both backward kernels run two warpgroups (256 threads): thread t owns TMEM
// lane / tile row t % 128 and the column half t / 128 of every 64-wide row,
// so the elementwise work and the running sums are split between them.
//
// Accumulation. The tensor cores' fp32 accumulation is not rounded to
// nearest: adding several hundred MMA steps into one TMEM accumulator (a
// head of 1024 queries gives 16 tiles x 24 steps) drifts by about 1e-5 of
// the result. So the MMAs of one streamed tile start a fresh partial sum in
// TMEM (24 steps), and the threads add the partials into registers with
// ordinary round-to-nearest fp32 adds.
constexpr int kBwdThreads = 256;

// 32 values into the three pieces in TMEM at taddr (piece a at +32 a), 16
// values (8 columns) at a time.
__device__ __forceinline__ void split32_to_tmem(const uint32_t (&v)[32], uint32_t taddr) {
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
        uint32_t w0[8], w1[8], w2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            split2(__uint_as_float(v[16 * qq + 2 * e]), __uint_as_float(v[16 * qq + 2 * e + 1]),
                   w0[e], w1[e], w2[e]);
        tmem_st8(taddr + 8 * qq, w0);
        tmem_st8(taddr + 8 * qq + 32, w1);
        tmem_st8(taddr + 8 * qq + 64, w2);
    }
}


// acc[0..31] += the 32 fp32 columns of this lane at taddr. The tiles' dV,
// dK and dQ are summed here in fp32 rather than by accumulating MMAs across
// tiles in TMEM, which measured above the fp32 parity bar.
__device__ __forceinline__ void add_tmem32(uint32_t taddr, float (&acc)[32]) {
    uint32_t r[32];
    tmem_ld32(taddr, r);
    tmem_ld_wait(r);
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] += __uint_as_float(r[c]);
}

// ---------------------------------------------------- dK and dV pass
// TMEM columns: S^T (64), dP^T (64), this tile's dV (64) and dK (64), P^T
// pieces (96), dS^T pieces (96).
constexpr uint32_t kKvColS = 0, kKvColdP = 64, kKvColdV = 128, kKvColdK = 192, kKvColP = 256,
                   kKvColdS = 352, kKvTmemCols = 512;
constexpr int kKvOffK = 0;
constexpr int kKvOffV = kKvOffK + kBigTile;
constexpr int kKvOffQ = kKvOffV + kBigTile;            // two buffers
constexpr int kKvOffdO = kKvOffQ + 2 * kSmallTile;     // two buffers
constexpr int kKvOffRow = kKvOffdO + 2 * kSmallTile;   // [2][LSE 64 | D 64] floats
constexpr int kKvOffStage = kKvOffRow + 4 * kSmall * 4; // Q, dO, LSE | D of tile t + 2
constexpr int kKvOffBar = kKvOffStage + 2 * kStageBytes + 2 * kSmall * 4;
constexpr int kKvSmemBytes = kKvOffBar + 128;

// CTA `cta` of the pass: one per (128-key tile, head), heads fastest; causal
// passes start with the first key tiles (the most query tiles).
__device__ __forceinline__ void
kv_pass(int cta, const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
        const float* __restrict__ dO, const float* __restrict__ lse2,
        const float* __restrict__ Dd, int n_pad, float* __restrict__ dK,
        float* __restrict__ dV, int n, int m, int d, int dv, int BH, int causal, float scale,
        float scale_log2, const int* __restrict__ key_len, int H,
        unsigned long long budget_ns) {
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + kKvOffBar);
    float* sRow = reinterpret_cast<float*>(smem + kKvOffRow);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane128 = tid & 127, half = tid >> 7;
    const int bh = cta % BH;
    const int kt = cta / BH;
    const int k0 = kt * kBig, krow = k0 + lane128;
    const float* Qh = Q + size_t(bh) * n * d;
    const float* Kh = K + size_t(bh) * m * d;
    const float* Vh = V + size_t(bh) * m * dv;
    const float* dOh = dO + size_t(bh) * n * dv;
    const float* L2h = lse2 + size_t(bh) * n_pad;
    const float* Dh = Dd + size_t(bh) * n_pad;
    const int nqs = (n + kSmall - 1) / kSmall;
    const int i0 = causal ? k0 / kSmall : 0;
    // Keys past mk are padding: their rows get P = 0 and zero dK, dV; a tile
    // of only padded keys visits one query tile so that the zeros are written.
    const int mk = keys_valid(key_len, bh, H, m);
    const bool key_dead = krow >= mk;
    const int T = (k0 >= mk) ? 1 : nqs - i0;   // >= 1: causal has n == m > k0

    // rows < n_pad: 64-row tiles never pass the 128-row padding
    auto load_q = [&](int idx, int buf) {
        const int r0 = (i0 + idx) * kSmall;
        load_split2<kSmall, kBwdThreads>(Qh, d, smem + kKvOffQ + buf * kSmallTile, dOh, dv,
                                         smem + kKvOffdO + buf * kSmallTile, r0, n, tid);
        if (tid < kSmall) sRow[buf * 128 + tid] = L2h[r0 + tid];
        else if (tid < 2 * kSmall) sRow[buf * 128 + tid] = Dh[r0 + tid - kSmall];
    };
    uint8_t* stQ = smem + kKvOffStage;
    uint8_t* stdO = stQ + kStageBytes;
    uint8_t* stRow = stdO + kStageBytes;                 // LSE 64 | D 64 floats
    auto fetch_q = [&](int idx) {
        const int r0 = (i0 + idx) * kSmall;
        fetch<kSmall, kBwdThreads>(Qh, r0, n, d, stQ, tid);
        fetch<kSmall, kBwdThreads>(dOh, r0, n, dv, stdO, tid);
        if (tid < 16) cp_async16(stRow + 16 * tid, L2h + r0 + 4 * tid, 16);
        else if (tid < 32) cp_async16(stRow + 16 * tid, Dh + r0 + 4 * (tid - 16), 16);
        cp_async_commit();
    };
    auto split_q = [&](int buf) {
        split_staged<kSmall, kBwdThreads>(stQ, smem + kKvOffQ + buf * kSmallTile, tid);
        split_staged<kSmall, kBwdThreads>(stdO, smem + kKvOffdO + buf * kSmallTile, tid);
        if (tid < 32)
            *reinterpret_cast<float4*>(sRow + buf * 128 + 4 * tid) =
                *reinterpret_cast<const float4*>(stRow + 16 * tid);
    };

    init_bars(bars, kKvTmemCols);
    const bool aligned = (smem_addr(smem) & 1023u) == 0;
    if (aligned) {
        // Query tiles 0 and 1 are split in place; tile 2 is in flight meanwhile.
        if (T > 2) fetch_q(2);
        load_split2<kBig, kBwdThreads>(Kh, d, smem + kKvOffK, Vh, dv, smem + kKvOffV, k0, m, tid);
        load_q(0, 0);
        if (T > 1) load_q(1, 1);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tl = tmem + (uint32_t((warp & 3) * 32) << 16) + 32 * half;
    const uint32_t sK = smem_addr(smem + kKvOffK), sV = smem_addr(smem + kKvOffV);
    const uint32_t sQ = smem_addr(smem + kKvOffQ), sdO = smem_addr(smem + kKvOffdO);
    const int never = 0;

    bool ok = aligned;
    if (!aligned && tid == 0) record_device_error(kErrTimeout);
    if (ok && tid == 0) {
        mma6_ss(tmem + kKvColS, sK, kBigPiece, sQ, kSmallPiece, kIdSS);
        mma6_ss(tmem + kKvColdP, sV, kBigPiece, sdO, kSmallPiece, kIdSS);
        mma_commit(&bars->bar_a);
    }

    // Per query tile: S^T/dP^T(idx) -> P^T, dS^T in registers -> (once the
    // previous tile's dV/dK MMAs are done with the pieces) split into TMEM ->
    // S^T/dP^T(idx+1), then dV/dK(idx). S^T/dP^T of the next tile are issued
    // first, so the P/dS arithmetic of tile idx+1 runs under the dV/dK MMAs
    // of tile idx; each tile's dV and dK are added into registers.
    float acc_v[32], acc_k[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc_v[c] = acc_k[c] = 0.f;
    for (int idx = 0; ok && idx < T; ++idx) {
        const int buf = idx & 1;
        const int qb = (i0 + idx) * kSmall + 32 * half;     // first query of this half
        bool got = mbar_wait_warp(&bars->bar_a, idx & 1, &never, budget_ns);
        uint32_t sr[32], pr[32];
        if (got) {
            tc_fence_after();
            const float* Lrow = sRow + buf * 128 + 32 * half;
            const float* Drow = Lrow + kSmall;
            tmem_ld32(tl + kKvColS, sr);
            tmem_ld32(tl + kKvColdP, pr);
            tmem_ld_wait(sr);
            tmem_ld_wait(pr);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                float pv = ex2(fmaf(__uint_as_float(sr[c]), scale_log2, -Lrow[c]));
                if (key_dead || (causal && krow > qb + c)) pv = 0.f;
                sr[c] = __float_as_uint(pv);
                pr[c] = __float_as_uint(pv * fmaf(__uint_as_float(pr[c]), scale, -Drow[c]));
            }
        }
        // The previous tile's dV/dK MMAs have read the P^T/dS^T pieces and
        // Q, dO of buffer buf^1: tile idx + 1 goes there, idx + 2 starts
        // arriving.
        if (got && idx > 0) {
            got = mbar_wait_warp(&bars->bar_b, (idx - 1) & 1, &never, budget_ns);
            if (got) {
                tc_fence_after();
                add_tmem32(tl + kKvColdV, acc_v);
                add_tmem32(tl + kKvColdK, acc_k);
            }
            if (got && idx + 1 < T) {
                split_q(buf ^ 1);
                fence_proxy_async_smem();
                if (idx + 2 < T) fetch_q(idx + 2);
            }
        }
        if (got) {
            // this half's 32 queries are K elements 32 half .. +31: columns 16 half ..
            split32_to_tmem(sr, tl - 32 * half + kKvColP + 16 * half);
            split32_to_tmem(pr, tl - 32 * half + kKvColdS + 16 * half);
            tmem_st_wait();
        }
        tc_fence_before();
        if (__syncthreads_or(!got)) {
            ok = false;
            break;
        }
        if (tid == 0) {
            tc_fence_after();
            if (idx + 1 < T) {
                mma6_ss(tmem + kKvColS, sK, kBigPiece, sQ + (buf ^ 1) * kSmallTile, kSmallPiece,
                        kIdSS);
                mma6_ss(tmem + kKvColdP, sV, kBigPiece, sdO + (buf ^ 1) * kSmallTile, kSmallPiece,
                        kIdSS);
                mma_commit(&bars->bar_a);
            }
            mma6_ts(tmem + kKvColdV, tmem + kKvColP, sdO + buf * kSmallTile, kIdTS, false);
            mma6_ts(tmem + kKvColdK, tmem + kKvColdS, sQ + buf * kSmallTile, kIdTS, false);
            mma_commit(&bars->bar_b);
        }
    }

    if (ok) {
        ok = mbar_wait_warp(&bars->bar_b, (T - 1) & 1, &never, budget_ns);
        if (ok) {
            tc_fence_after();
            add_tmem32(tl + kKvColdV, acc_v);
            add_tmem32(tl + kKvColdK, acc_k);
            if (krow < m) {
                store_half(dV + (size_t(bh) * m + krow) * dv, 32 * half, acc_v, dv);
                store_half(dK + (size_t(bh) * m + krow) * d, 32 * half, acc_k, d);
            }
        }
    }
    if (!ok && tid == 0) record_device_error(kErrTimeout);
    teardown(bars, tmem, kKvTmemCols, budget_ns);
}

// ----------------------------------------------------------- dQ pass
// TMEM columns: S (64), dP (64), this tile's dQ (64), dS pieces (96).
constexpr uint32_t kDqColS = 0, kDqColdP = 64, kDqColdQ = 128, kDqColdS = 192, kDqTmemCols = 512;
constexpr int kDqOffQ = 0;
constexpr int kDqOffdO = kDqOffQ + kBigTile;
constexpr int kDqOffK = kDqOffdO + kBigTile;           // two buffers
constexpr int kDqOffV = kDqOffK + 2 * kSmallTile;      // two buffers
constexpr int kDqOffStage = kDqOffV + 2 * kSmallTile;  // K, V of tile t + 2
constexpr int kDqOffBar = kDqOffStage + 2 * kStageBytes;
constexpr int kDqSmemBytes = kDqOffBar + 128;

// CTA `cta` of the pass: one per (128-query tile, head), ordered as the
// forward's CTAs.
__device__ __forceinline__ void
dq_pass(int cta, const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
        const float* __restrict__ dO, const float* __restrict__ lse2,
        const float* __restrict__ Dd, int n_pad, float* __restrict__ dQ, int n, int m, int d,
        int dv, int BH, int causal, float scale, float scale_log2,
        const int* __restrict__ key_len, int H, unsigned long long budget_ns) {
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem + kDqOffBar);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane128 = tid & 127, half = tid >> 7;
    const int num_qt = (n + kBig - 1) / kBig;
    const int bh = cta % BH;
    const int rank = cta / BH;
    const int qt = causal ? num_qt - 1 - rank : rank;
    const int q0 = qt * kBig, row = q0 + lane128;
    const float* Qh = Q + size_t(bh) * n * d;
    const float* Kh = K + size_t(bh) * m * d;
    const float* Vh = V + size_t(bh) * m * dv;
    const float* dOh = dO + size_t(bh) * n * dv;
    const float l2 = lse2[size_t(bh) * n_pad + row];     // row < n_pad
    const float dd = Dd[size_t(bh) * n_pad + row];
    const int mk = keys_valid(key_len, bh, H, m);        // keys past mk: padding
    const int nkt = (mk + kSmall - 1) / kSmall;
    const int T = causal ? min(nkt, (q0 + kBig - 1) / kSmall + 1) : nkt;

    uint8_t* stK = smem + kDqOffStage;
    uint8_t* stV = stK + kStageBytes;
    auto fetch_kv = [&](int t) {
        fetch<kSmall, kBwdThreads>(Kh, t * kSmall, m, d, stK, tid);
        fetch<kSmall, kBwdThreads>(Vh, t * kSmall, m, dv, stV, tid);
        cp_async_commit();
    };

    init_bars(bars, kDqTmemCols);
    const bool aligned = (smem_addr(smem) & 1023u) == 0;
    if (aligned) {
        // Key tiles 0 and 1 are split in place; tile 2 is in flight meanwhile.
        if (T > 2) fetch_kv(2);
        load_split2<kBig, kBwdThreads>(Qh, d, smem + kDqOffQ, dOh, dv, smem + kDqOffdO, q0, n, tid);
        load_split2<kSmall, kBwdThreads>(Kh, d, smem + kDqOffK, Vh, dv, smem + kDqOffV, 0, m, tid);
        if (T > 1) {
            load_split2<kSmall, kBwdThreads>(Kh, d, smem + kDqOffK + kSmallTile, Vh, dv,
                                             smem + kDqOffV + kSmallTile, kSmall, m, tid);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tl = tmem + (uint32_t((warp & 3) * 32) << 16) + 32 * half;
    const uint32_t sQ = smem_addr(smem + kDqOffQ), sdO = smem_addr(smem + kDqOffdO);
    const uint32_t sK = smem_addr(smem + kDqOffK), sV = smem_addr(smem + kDqOffV);
    const int never = 0;

    bool ok = aligned;
    if (!aligned && tid == 0) record_device_error(kErrTimeout);
    if (ok && tid == 0) {
        mma6_ss(tmem + kDqColS, sQ, kBigPiece, sK, kSmallPiece, kIdSS);
        mma6_ss(tmem + kDqColdP, sdO, kBigPiece, sV, kSmallPiece, kIdSS);
        mma_commit(&bars->bar_a);
    }

    // Per key tile, as in the dK/dV pass: S/dP(j) -> dS in registers ->
    // (once dQ(j-1) has read the dS pieces and K of buffer buf^1) split into
    // TMEM -> S/dP(j+1), then dQ(j); each tile's dQ is added into registers.
    float acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = 0.f;
    for (int j = 0; ok && j < T; ++j) {
        const int buf = j & 1;
        const int kb = j * kSmall + 32 * half;               // first key of this half
        bool got = mbar_wait_warp(&bars->bar_a, j & 1, &never, budget_ns);
        uint32_t pr[32];
        if (got) {
            tc_fence_after();
            uint32_t sr[32];
            tmem_ld32(tl + kDqColS, sr);
            tmem_ld32(tl + kDqColdP, pr);
            tmem_ld_wait(sr);
            tmem_ld_wait(pr);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const int key = kb + c;
                float pv = ex2(fmaf(__uint_as_float(sr[c]), scale_log2, -l2));
                if (key >= mk || (causal && key > row)) pv = 0.f;
                pr[c] = __float_as_uint(pv * fmaf(__uint_as_float(pr[c]), scale, -dd));
            }
        }
        // K, V of buffer buf^1 (tile j-1) and the dS pieces are free once
        // dQ(j-1) is done: tile j + 1 goes there, j + 2 starts arriving.
        if (got && j > 0) {
            got = mbar_wait_warp(&bars->bar_b, (j - 1) & 1, &never, budget_ns);
            if (got) {
                tc_fence_after();
                add_tmem32(tl + kDqColdQ, acc);
            }
            if (got && j + 1 < T) {
                split_staged<kSmall, kBwdThreads>(stK, smem + kDqOffK + (buf ^ 1) * kSmallTile, tid);
                split_staged<kSmall, kBwdThreads>(stV, smem + kDqOffV + (buf ^ 1) * kSmallTile, tid);
                fence_proxy_async_smem();
                if (j + 2 < T) fetch_kv(j + 2);
            }
        }
        if (got) {
            split32_to_tmem(pr, tl - 32 * half + kDqColdS + 16 * half);
            tmem_st_wait();
        }
        tc_fence_before();
        if (__syncthreads_or(!got)) {
            ok = false;
            break;
        }
        if (tid == 0) {
            tc_fence_after();
            if (j + 1 < T) {
                mma6_ss(tmem + kDqColS, sQ, kBigPiece, sK + (buf ^ 1) * kSmallTile, kSmallPiece,
                        kIdSS);
                mma6_ss(tmem + kDqColdP, sdO, kBigPiece, sV + (buf ^ 1) * kSmallTile, kSmallPiece,
                        kIdSS);
                mma_commit(&bars->bar_a);
            }
            mma6_ts(tmem + kDqColdQ, tmem + kDqColdS, sK + buf * kSmallTile, kIdTS, false);
            mma_commit(&bars->bar_b);
        }
    }

    if (ok) {
        ok = mbar_wait_warp(&bars->bar_b, (T - 1) & 1, &never, budget_ns);
        if (ok) {
            tc_fence_after();
            add_tmem32(tl + kDqColdQ, acc);
            if (row < n) store_half(dQ + (size_t(bh) * n + row) * d, 32 * half, acc, d);
        }
    }
    if (!ok && tid == 0) record_device_error(kErrTimeout);
    teardown(bars, tmem, kDqTmemCols, budget_ns);
}

// ------------------------------------------------------- one launch
// Both passes in one grid: CTAs [0, kv_ctas) run the dK/dV pass and the rest
// the dQ pass. The passes share no data, and one launch lets each pass's
// last, partial wave of CTAs be filled by the other's.
constexpr int kBwdSmemBytes = kKvSmemBytes > kDqSmemBytes ? kKvSmemBytes : kDqSmemBytes;

__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_kernel(const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
           const float* __restrict__ dO, const float* __restrict__ lse2,
           const float* __restrict__ Dd, int n_pad, float* __restrict__ dQ,
           float* __restrict__ dK, float* __restrict__ dV, int n, int m, int d, int dv, int BH,
           int causal, float scale, float scale_log2, const int* __restrict__ key_len, int H,
           int kv_ctas, unsigned long long budget_ns) {
    const int b = int(blockIdx.x);
    if (b < kv_ctas)
        kv_pass(b, Q, K, V, dO, lse2, Dd, n_pad, dK, dV, n, m, d, dv, BH, causal, scale,
                scale_log2, key_len, H, budget_ns);
    else
        dq_pass(b - kv_ctas, Q, K, V, dO, lse2, Dd, n_pad, dQ, n, m, d, dv, BH, causal, scale,
                scale_log2, key_len, H, budget_ns);
}

}  // namespace f32x
}  // namespace attn
