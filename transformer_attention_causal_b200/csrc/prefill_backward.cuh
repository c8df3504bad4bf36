// Backward pass of full-sequence attention on the 5th-generation tensor cores.
//
// The forward saves one statistic per query row, lse = m + ln(l) (the row
// maximum and exponential sum folded into one number), and the backward
// rebuilds every probability it needs from Q, K and that statistic, so no
// T x T matrix is ever stored ("Causal Multi-Head Self-Attention", Two exact
// full-sequence algorithms: the Flash path keeps only the row statistics and
// recomputes probabilities tile by tile, then applies the exact softmax
// vector-Jacobian product).  With s = scale * q.k, P = exp(s - lse) on the
// visible keys (0 on masked ones) and the upstream gradient dO:
//
//   D_i  = sum_t dO_it O_it            (= sum_j P_ij dP_ij, the row term)
//   dP   = dO V^T,   dS = P o (dP - D)
//   dV   = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K
//
// Three kernels, all on the caller's stream:
//   bwd_preprocess   D and -lse*log2(e) per row into the workspace, padded to
//                    whole 128-row tiles (-inf / 0 on the padding, so padded
//                    query rows carry P = 0 without a mask);
//   bwd_dkdv         one CTA per (batch, K/V head, 128-key tile): loops over
//                    the G query heads of the K/V head and the query tiles
//                    that see the keys, so dK and dV of grouped heads are
//                    summed in TMEM, not with atomics ("Grouped-Query
//                    Attention" §5.1);
//   bwd_dq           one CTA per (batch, head, 128-query tile): loops over
//                    the key tiles the rows see.
// In both tensor-core kernels warp 0 is the TMA producer, warp 1 owns TMEM
// and issues the MMAs from one thread, warps 4-11 do the elementwise work:
// one TMEM lane (a key row in bwd_dkdv, a query row in bwd_dq) per thread,
// warps 4-7 on the tile's columns 0-63 and warps 8-11 on columns 64-127 (no
// step of the backward reduces along a row, so the halves never meet).
// 16-bit P / dS values of columns 64h..64h+63 are packed into TMEM columns
// 64h..64h+31 of the region they were read from, so a half never overwrites
// scores the other half has yet to read; the TS MMAs' A operand follows that
// map (k-steps 4-7 start 32 columns further on).
//
// bwd_dkdv, TMEM columns: S^T [0,128), dP^T [128,256), dV [256,384),
// dK [384,512).  Per query tile:
//   S^T = K Q^T, dP^T = V dO^T        (SS MMAs, M = N = 128)
//   P^T (16-bit) over the first 64 columns of S^T  -> dV += P^T dO  (TS MMA)
//   dS^T (16-bit) over the first 64 columns of dP^T -> dK += dS^T Q  (TS MMA)
// Issue order: dV(t), S^T(t+1), dK(t), dP^T(t+1): each overwrite of a TMEM
// region follows the MMA that read it, and the next tile's exponentials
// overlap this tile's dK and the next dP^T.
//
// bwd_dq, TMEM columns: S [0,128), dP [128,256), dQ [256,256+d), dS (16-bit
// pairs) [384,448), Q (16-bit pairs, copied in once by the elementwise warps)
// [448,512).  Per key tile: S = Q K^T (TS: Q from TMEM), dP = dO V^T (SS),
// dQ += dS K (TS).  Every shared-memory operand read competes with the TMA
// copies for the SM's 128 B/clk, so Q comes from TMEM; and because dS has
// its own columns, S(n+1) and dP(n+1) are issued as soon as the elementwise
// warps have read S(n) and dP(n) into registers.
#pragma once

#include "prefill_tcgen05.cuh"

namespace b200attn {

struct BwdParams {
    const void* o;
    const void* dout;
    const float* lse;     // [B*H, T] natural-log row statistic from the forward
    void* dq;             // [B, H, T, d]
    void* dk;             // [B, Hkv, T, d]
    void* dv;             // [B, Hkv, T, d]
    float* nl;            // workspace [B*H, Tpad]: -lse * log2(e); -inf on padding rows
    float* dd;            // workspace [B*H, Tpad]: D = sum_t dO*O; 0 on padding rows
    int B, H, Hkv, G, T, Tpad, d, causal;
    int window;           // local window w (causal): row i reads keys i - w < j <= i; 0: none
    int n_t;              // ceil(T / 128)
    int group_kv, group_q; // work order (grouped_order): items per L2 group, dK/dV and dQ kernels
    float scale, scale_log2;
    uint64_t timeout_ns;
    uint32_t test_flags;  // kTestSkipLoads: issue no copies (timeout-path tests)
};

constexpr int kBwdThreads = 384;  // 12 warps: producer, MMA, 2 idle, 8 elementwise

// Ring depths, as deep as shared memory allows.  In bwd_dq a K tile is read
// from S(n) until dQ(n), a V tile only by dP(n): separate rings, the K ring
// the deeper.
template <int DCH> struct BwdStages {
    static constexpr int NQ = DCH == 2 ? 2 : 5;    // bwd_dkdv: (Q, dO, nl, D) stages
    static constexpr int NKR = DCH == 2 ? 3 : 6;   // bwd_dq: K stages (read by S(n) and dQ(n))
    static constexpr int NVR = DCH == 2 ? 2 : 4;   // bwd_dq: V stages (read by dP(n) only)
};

template <int DCH>
constexpr size_t bwd_dkdv_smem_bytes() {
    return 1024 + size_t(2 + 2 * BwdStages<DCH>::NQ) * DCH * kChunkBytes +
           size_t(BwdStages<DCH>::NQ) * 1024 + 256;
}

template <int DCH>
constexpr size_t bwd_dq_smem_bytes() {
    return 1024 + size_t(2 + BwdStages<DCH>::NKR + BwdStages<DCH>::NVR) * DCH * kChunkBytes + 256;
}

// ------------------------------------------------------------------ preprocess

// D and -lse*log2(e) for every row of [B*H, Tpad]; one half-warp per row
// (16 lanes x 8 elements cover d <= 128).
template <typename T>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BwdParams p) {
    const int64_t rows = int64_t(p.B) * p.H * p.Tpad;
    const int half = threadIdx.x >> 4;
    const int hl = threadIdx.x & 15;
    // the loop bound is uniform over the block, so every shuffle has all lanes
    for (int64_t r0 = int64_t(blockIdx.x) * 16; r0 < rows; r0 += int64_t(gridDim.x) * 16) {
        const int64_t r = r0 + half;
        const bool live = r < rows;
        const int64_t bh = live ? r / p.Tpad : 0;
        const int i = live ? int(r - bh * p.Tpad) : p.T;
        float acc = 0.f;
        if (i < p.T) {
            const size_t off = (size_t(bh) * p.T + i) * p.d;
            const T* o = static_cast<const T*>(p.o) + off;
            const T* g = static_cast<const T*>(p.dout) + off;
            for (int c = hl * 8; c < p.d; c += 128) {
                const uint4 a = *reinterpret_cast<const uint4*>(o + c);
                const uint4 b = *reinterpret_cast<const uint4*>(g + c);
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack2<T>(aw[e]), y = unpack2<T>(bw[e]);
                    acc = fmaf(x.x, y.x, acc);
                    acc = fmaf(x.y, y.y, acc);
                }
            }
        }
#pragma unroll
        for (int m = 8; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        if (live && hl == 0) {
            p.dd[r] = i < p.T ? acc : 0.f;
            p.nl[r] = i < p.T ? -p.lse[size_t(bh) * p.T + i] * 1.4426950408889634f : -INFINITY;
        }
    }
}

// ------------------------------------------------------------------ MMA helpers

// D (128 x 128, fp32 in TMEM) = A B^T with both operands K-major 128-row
// tiles in shared memory (d/16 k-steps over the DCH 64-column chunks).
template <int DCH>
__device__ __forceinline__ void bwd_mma_rows(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                             int nk) {
#pragma unroll
    for (int kk = 0; kk < 4 * DCH; ++kk) {
        if (kk >= nk) break;
        const uint64_t off = uint64_t(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
        mma_ss(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
    }
}

// D (128 x d) (+)= A B with A (128 x 128, 16-bit) in TMEM and B a 128-row tile
// in shared memory read MN-major (rows are the contraction index).  A's
// contraction columns 0-63 sit in TMEM columns 0-31, columns 64-127 in TMEM
// columns 64-95 (each elementwise half packs into its own range).
__device__ __forceinline__ void bwd_mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0,
                                               uint32_t idesc, bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_ts(d_tmem, a_tmem + kk * 8 + (kk >= 4 ? 32 : 0), b0 + uint64_t((kk * 2048) >> 4), idesc,
               (accumulate || kk > 0) ? 1u : 0u);
}

// 32 consecutive fp32 values of shared memory (16-byte aligned shared
// address) into registers, 16 bytes per load (every lane reads the same
// address: one broadcast per load).
__device__ __forceinline__ void lds32(uint32_t saddr, float (&r)[32]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(r[4 * i]), "=f"(r[4 * i + 1]), "=f"(r[4 * i + 2]), "=f"(r[4 * i + 3])
                     : "r"(saddr + 16 * i));
}

// One tile row's epilogue: 16-column pieces first, first + step, ... of a
// TMEM accumulator, times `mul`, rounded to T and stored to `dst` (d
// elements) when `valid`.
template <typename T>
__device__ __forceinline__ void bwd_store_row(uint32_t t_acc, int d, float mul, T* dst, bool valid,
                                              int first = 0, int step = 16) {
    for (int cc = first; cc < d; cc += step) {
        uint32_t x[16];
        tmem_ld16(t_acc + cc, x);
        tmem_wait_ld();
        uint4 w0, w1;
        w0.x = pack2<T>(__uint_as_float(x[0]) * mul, __uint_as_float(x[1]) * mul);
        w0.y = pack2<T>(__uint_as_float(x[2]) * mul, __uint_as_float(x[3]) * mul);
        w0.z = pack2<T>(__uint_as_float(x[4]) * mul, __uint_as_float(x[5]) * mul);
        w0.w = pack2<T>(__uint_as_float(x[6]) * mul, __uint_as_float(x[7]) * mul);
        w1.x = pack2<T>(__uint_as_float(x[8]) * mul, __uint_as_float(x[9]) * mul);
        w1.y = pack2<T>(__uint_as_float(x[10]) * mul, __uint_as_float(x[11]) * mul);
        w1.z = pack2<T>(__uint_as_float(x[12]) * mul, __uint_as_float(x[13]) * mul);
        w1.w = pack2<T>(__uint_as_float(x[14]) * mul, __uint_as_float(x[15]) * mul);
        if (valid) {
            reinterpret_cast<uint4*>(dst + cc)[0] = w0;
            reinterpret_cast<uint4*>(dst + cc)[1] = w1;
        }
    }
}

// ------------------------------------------------------------------ dK, dV

template <typename T, int DCH, bool WINDOW>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                const BwdParams p) {
    constexpr int NQ = BwdStages<DCH>::NQ;
    constexpr uint32_t TB = DCH * kChunkBytes;   // one 128-row tile
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char* base_ptr = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t sK = base, sV = base + TB;
    const uint32_t sQ = base + 2 * TB;              // [NQ] tiles
    const uint32_t sdO = sQ + NQ * TB;              // [NQ] tiles
    float* rowstat = reinterpret_cast<float*>(base_ptr + (2 + 2 * NQ) * TB);  // [NQ][nl 128 | D 128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(rowstat + NQ * 256);
    uint64_t* kv_full = bars;            // 1
    uint64_t* q_full = bars + 1;         // NQ
    uint64_t* q_empty = q_full + NQ;     // NQ: the MMA commit + 8 elementwise warps
    uint64_t* s_full = q_empty + NQ;     // 1
    uint64_t* dp_full = s_full + 1;      // 1
    uint64_t* p_ready = dp_full + 1;     // 1 (8 arrivals)
    uint64_t* ds_ready = p_ready + 1;    // 1 (8 arrivals)
    uint64_t* acc_done = ds_ready + 1;   // 1
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // (b, K/V head) in groups whose Q and dO tiles fit in L2 together, each
    // group heaviest (kt = 0) first
    int kt, bk;
    grouped_order(blockIdx.x, p.B * p.Hkv, p.n_t, p.group_kv, kt, bk);
    const int b = bk / p.Hkv, kvh = bk % p.Hkv;
    const int q_lo = p.causal ? kt : 0;
    // with a window only the query tiles whose rows reach this key tile
    const int q_hi = WINDOW ? min(p.n_t - 1, (kt * 128 + 127 + p.window - 1) / 128) : p.n_t - 1;
    const int n_q = q_hi - q_lo + 1;
    const int n_it = p.G * n_q;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(kv_full), 1);
        for (int s = 0; s < NQ; ++s) {
            mbar_init(smem_u32(&q_full[s]), 1);
            mbar_init(smem_u32(&q_empty[s]), 9);
        }
        mbar_init(smem_u32(s_full), 1);
        mbar_init(smem_u32(dp_full), 1);
        mbar_init(smem_u32(p_ready), 8);
        mbar_init(smem_u32(ds_ready), 8);
        mbar_init(smem_u32(acc_done), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0) {
            const bool skip = p.test_flags & kTestSkipLoads;
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmdO);
            if (!skip) {
                const uint32_t bar = smem_u32(kv_full);
                mbar_expect_tx(bar, 2 * TB);
                for (int c = 0; c < DCH; ++c) {
                    tma_load_3d(sK + c * kChunkBytes, &tmK, bar, c * 64, kt * 128, bk);
                    tma_load_3d(sV + c * kChunkBytes, &tmV, bar, c * 64, kt * 128, bk);
                }
            }
            int it = 0;
            for (; it < n_it && !skip; ++it) {
                const int st = it % NQ;
                if (!mbar_wait(smem_u32(&q_empty[st]), ((it / NQ) & 1) ^ 1, p.timeout_ns, abort_flag)) break;
                const int h = kvh * p.G + it / n_q;
                const int qt = q_lo + it % n_q;
                const int bh = b * p.H + h;
                const uint32_t bar = smem_u32(&q_full[st]);
                mbar_expect_tx(bar, 2 * TB + 1024);
                for (int c = 0; c < DCH; ++c) {
                    tma_load_3d(sQ + st * TB + c * kChunkBytes, &tmQ, bar, c * 64, qt * 128, bh);
                    tma_load_3d(sdO + st * TB + c * kChunkBytes, &tmdO, bar, c * 64, qt * 128, bh);
                }
                const size_t ro = size_t(bh) * p.Tpad + size_t(qt) * 128;
                bulk_load(smem_u32(rowstat + st * 256), p.nl + ro, 512, bar);
                bulk_load(smem_u32(rowstat + st * 256 + 128), p.dd + ro, 512, bar);
            }
            // no copy may still be landing when the CTA exits
            if (!skip) mbar_wait(smem_u32(kv_full), 0, p.timeout_ns, nullptr);
            for (int i = it - 1; i >= 0 && i >= it - NQ; --i)
                mbar_wait(smem_u32(&q_full[i % NQ]), (i / NQ) & 1, p.timeout_ns, nullptr);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_f16(kBF16, 128, 128, false);
            const uint32_t idA = idesc_f16(kBF16, 128, p.d, true);
            const int nk = p.d / 16;
            const uint64_t aK = smem_desc_sw128(sK, 16, 1024);
            const uint64_t aV = smem_desc_sw128(sV, 16, 1024);
            const uint64_t bQk = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t bdOk = smem_desc_sw128(sdO, 16, 1024);
            const uint64_t bQm = smem_desc_sw128(sQ, kChunkBytes, 1024);
            const uint64_t bdOm = smem_desc_sw128(sdO, kChunkBytes, 1024);
            const auto step = [](int st) { return uint64_t(uint32_t(st) * (TB >> 4)); };
            bool ok = mbar_wait(smem_u32(kv_full), 0, p.timeout_ns, abort_flag);
            if (ok) ok = mbar_wait(smem_u32(&q_full[0]), 0, p.timeout_ns, abort_flag);
            if (ok) {
                tc_fence_after();
                bwd_mma_rows<DCH>(tmem, aK, bQk, idS, nk);
                mma_commit(smem_u32(s_full));
                bwd_mma_rows<DCH>(tmem + 128, aV, bdOk, idS, nk);
                mma_commit(smem_u32(dp_full));
            }
            for (int it = 0; it < n_it && ok; ++it) {
                const int st = it % NQ;
                const int st1 = (it + 1) % NQ;
                const bool more = it + 1 < n_it;
                ok = mbar_wait(smem_u32(p_ready), it & 1, p.timeout_ns, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bwd_mma_tmem_a(tmem + 256, tmem, bdOm + step(st), idA, it > 0);
                if (more) {
                    ok = mbar_wait(smem_u32(&q_full[st1]), ((it + 1) / NQ) & 1, p.timeout_ns, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    bwd_mma_rows<DCH>(tmem, aK, bQk + step(st1), idS, nk);
                    mma_commit(smem_u32(s_full));
                }
                ok = mbar_wait(smem_u32(ds_ready), it & 1, p.timeout_ns, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bwd_mma_tmem_a(tmem + 384, tmem + 128, bQm + step(st), idA, it > 0);
                mma_commit(smem_u32(&q_empty[st]));
                if (more) {
                    bwd_mma_rows<DCH>(tmem + 128, aV, bdOk + step(st1), idS, nk);
                    mma_commit(smem_u32(dp_full));
                }
            }
            // every MMA issued must finish before TMEM is released
            mma_commit(smem_u32(acc_done));
            mbar_wait(smem_u32(acc_done), 0, p.timeout_ns, nullptr);
        }
    } else if (warp >= 4) {
        // ================================================= elementwise (one key row per thread)
        const int wq = warp & 3;
        const int half = (warp - 4) >> 2;         // query columns 64*half .. 64*half + 63
        const int row = wq * 32 + lane;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + 64 * half, tdP = tmem + lane_base + 128 + 64 * half;
        const float c2 = p.scale_log2;
        bool ok = true;
        for (int it = 0; it < n_it && ok; ++it) {
            const int st = it % NQ;
            const int qt = q_lo + it % n_q;
            const uint32_t nl = smem_u32(rowstat + st * 256 + 64 * half);
            const uint32_t dd = nl + 128 * 4;
            ok = mbar_wait(smem_u32(s_full), it & 1, p.timeout_ns, abort_flag);
            if (ok) ok = mbar_wait(smem_u32(&q_full[st]), (it / NQ) & 1, p.timeout_ns, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[2][32];
            tmem_ld32(tS + 0, r[0]);
            tmem_ld32(tS + 32, r[1]);
            tmem_wait_ld();
            // causal diagonal tile: query column i sees key row j only when i >= j;
            // with a window also only while i - j < w
            const int rel = row - (qt - kt) * 128 - 64 * half;   // column of i = j in this half
            const int first_vis = (p.causal && qt == kt) ? rel : -64 * half - 1;
            const int end_vis = WINDOW ? rel + p.window : 64;
            const float2 c2v = make_float2(c2, c2);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                float nlv[32];
                lds32(nl + 128 * ch, nlv);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float2 x = __ffma2_rn(make_float2(__uint_as_float(r[ch][2 * e]),
                                                      __uint_as_float(r[ch][2 * e + 1])),
                                          c2v, make_float2(nlv[2 * e], nlv[2 * e + 1]));
                    if (32 * ch + 2 * e < first_vis) x.x = -INFINITY;
                    if (32 * ch + 2 * e + 1 < first_vis) x.y = -INFINITY;
                    if (WINDOW && 32 * ch + 2 * e >= end_vis) x.x = -INFINITY;
                    if (WINDOW && 32 * ch + 2 * e + 1 >= end_vis) x.y = -INFINITY;
                    const float p0 = ex2(x.x), p1 = ex2(x.y);
                    r[ch][2 * e] = __float_as_uint(p0);
                    r[ch][2 * e + 1] = __float_as_uint(p1);
                    pk[e] = pack2<T>(p0, p1);
                }
                // columns [16ch, 16ch+16) of this half were read with chunk 0
                tmem_st16(tS + 16 * ch, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(p_ready));
            ok = mbar_wait(smem_u32(dp_full), it & 1, p.timeout_ns, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t g[32];
                tmem_ld32(tdP + 32 * ch, g);
                tmem_wait_ld();
                float ddv[32];
                lds32(dd + 128 * ch, ddv);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 pp = make_float2(__uint_as_float(r[ch][2 * e]), __uint_as_float(r[ch][2 * e + 1]));
                    const float2 t = __fadd2_rn(make_float2(__uint_as_float(g[2 * e]), __uint_as_float(g[2 * e + 1])),
                                                make_float2(-ddv[2 * e], -ddv[2 * e + 1]));
                    const float2 ds = __fmul2_rn(pp, t);
                    pk[e] = pack2<T>(ds.x, ds.y);
                }
                // columns [16ch, 16ch+16) of this half were read with chunks <= ch
                tmem_st16(tdP + 16 * ch, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(ds_ready));
                mbar_arrive(smem_u32(&q_empty[st]));
            }
        }
        // ---- epilogue: dV and scale * dK rows of this key tile
        if (ok) ok = mbar_wait(smem_u32(acc_done), 0, p.timeout_ns, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const int j = kt * 128 + row;
            const bool valid = j < p.T;
            const size_t orow = (size_t(bk) * p.T + (valid ? j : 0)) * p.d;
            if (half == 0)
                bwd_store_row<T>(tmem + lane_base + 256, p.d, 1.f, static_cast<T*>(p.dv) + orow, valid);
            else
                bwd_store_row<T>(tmem + lane_base + 384, p.d, p.scale, static_cast<T*>(p.dk) + orow, valid);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ dQ

template <typename T, int DCH, bool WINDOW>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
              const BwdParams p) {
    constexpr int NKR = BwdStages<DCH>::NKR;
    constexpr int NVR = BwdStages<DCH>::NVR;
    constexpr uint32_t TB = DCH * kChunkBytes;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char* base_ptr = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t sQ = base, sdO = base + TB;
    const uint32_t sK = base + 2 * TB;              // [NKR] K tiles
    const uint32_t sV = sK + NKR * TB;              // [NVR] V tiles
    uint64_t* bars = reinterpret_cast<uint64_t*>(base_ptr + (2 + NKR + NVR) * TB);
    uint64_t* q_full = bars;             // 1
    uint64_t* k_full = bars + 1;         // NKR
    uint64_t* k_empty = k_full + NKR;    // NKR
    uint64_t* v_full = k_empty + NKR;    // NVR
    uint64_t* v_empty = v_full + NVR;    // NVR
    uint64_t* s_full = v_empty + NVR;    // 1
    uint64_t* dp_full = s_full + 1;      // 1
    uint64_t* s_read = dp_full + 1;      // 1 (8 arrivals): S(n) in registers
    uint64_t* dp_read = s_read + 1;      // 1 (8 arrivals): dP(n) in registers
    uint64_t* ds_ready = dp_read + 1;    // 1 (8 arrivals): dS(n) in TMEM
    uint64_t* ds_free = ds_ready + 1;    // 1: dQ(n) has read dS(n)
    uint64_t* q_tmem = ds_free + 1;      // 1 (8 arrivals): Q copied into TMEM
    uint64_t* acc_done = q_tmem + 1;     // 1
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // (b, head) in groups whose K and V tiles fit in L2 together, each group
    // heaviest (last query tile) first
    int lvl, bh;
    grouped_order(blockIdx.x, p.B * p.H, p.n_t, p.group_q, lvl, bh);
    const int qt = p.n_t - 1 - lvl;
    const int b = bh / p.H, h = bh % p.H;
    const int bk = b * p.Hkv + h / p.G;
    // key tiles n_first .. n_first + n_kv - 1 (with a window: from the first
    // key the tile's first row sees); loop counters run from 0
    const int n_first = WINDOW ? max(0, qt * 128 - p.window + 1) / 128 : 0;
    const int n_kv = (p.causal ? qt + 1 : p.n_t) - n_first;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(q_full), 1);
        for (int s = 0; s < NKR; ++s) {
            mbar_init(smem_u32(&k_full[s]), 1);
            mbar_init(smem_u32(&k_empty[s]), 1);
        }
        for (int s = 0; s < NVR; ++s) {
            mbar_init(smem_u32(&v_full[s]), 1);
            mbar_init(smem_u32(&v_empty[s]), 1);
        }
        mbar_init(smem_u32(s_full), 1);
        mbar_init(smem_u32(dp_full), 1);
        mbar_init(smem_u32(s_read), 8);
        mbar_init(smem_u32(dp_read), 8);
        mbar_init(smem_u32(ds_ready), 8);
        mbar_init(smem_u32(ds_free), 1);
        mbar_init(smem_u32(q_tmem), 8);
        mbar_init(smem_u32(acc_done), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0) {
            const bool skip = p.test_flags & kTestSkipLoads;
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            if (!skip) {
                const uint32_t bar = smem_u32(q_full);
                mbar_expect_tx(bar, 2 * TB);
                for (int c = 0; c < DCH; ++c) {
                    tma_load_3d(sQ + c * kChunkBytes, &tmQ, bar, c * 64, qt * 128, bh);
                    tma_load_3d(sdO + c * kChunkBytes, &tmdO, bar, c * 64, qt * 128, bh);
                }
            }
            // K_m and V_m into their own rings, in tile order
            int issued[2] = {0, 0};   // K and V copies issued
            bool kv_ok = !skip;
            for (int m = 0; m < n_kv && kv_ok; ++m) {
                for (int which = 0; which < 2 && kv_ok; ++which) {
                    const int nst = which ? NVR : NKR;
                    const int st = m % nst;
                    uint64_t* emp = which ? v_empty : k_empty;
                    uint64_t* ful = which ? v_full : k_full;
                    if (!mbar_wait(smem_u32(&emp[st]), ((m / nst) & 1) ^ 1, p.timeout_ns, abort_flag)) {
                        kv_ok = false;
                        break;
                    }
                    const uint32_t bar = smem_u32(&ful[st]);
                    mbar_expect_tx(bar, TB);
                    const uint32_t dst = (which ? sV : sK) + st * TB;
                    for (int c = 0; c < DCH; ++c)
                        tma_load_3d(dst + c * kChunkBytes, which ? &tmV : &tmK, bar, c * 64,
                                    (n_first + m) * 128, bk);
                    ++issued[which];
                }
            }
            // no copy may still be landing when the CTA exits
            if (!skip) mbar_wait(smem_u32(q_full), 0, p.timeout_ns, nullptr);
            for (int i = issued[0] - 1; i >= 0 && i >= issued[0] - NKR; --i)
                mbar_wait(smem_u32(&k_full[i % NKR]), (i / NKR) & 1, p.timeout_ns, nullptr);
            for (int i = issued[1] - 1; i >= 0 && i >= issued[1] - NVR; --i)
                mbar_wait(smem_u32(&v_full[i % NVR]), (i / NVR) & 1, p.timeout_ns, nullptr);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_f16(kBF16, 128, 128, false);
            const uint32_t idA = idesc_f16(kBF16, 128, p.d, true);
            const int nk = p.d / 16;
            const uint64_t adO = smem_desc_sw128(sdO, 16, 1024);
            const uint64_t bKk = smem_desc_sw128(sK, 16, 1024);
            const uint64_t bKm = smem_desc_sw128(sK, kChunkBytes, 1024);
            const uint64_t bVk = smem_desc_sw128(sV, 16, 1024);
            const auto step = [](int st) { return uint64_t(uint32_t(st) * (TB >> 4)); };
            const auto kfull = [&](int m) {
                return mbar_wait(smem_u32(&k_full[m % NKR]), (m / NKR) & 1, p.timeout_ns, abort_flag);
            };
            const auto vfull = [&](int m) {
                return mbar_wait(smem_u32(&v_full[m % NVR]), (m / NVR) & 1, p.timeout_ns, abort_flag);
            };
            // S(m) = Q K_m^T with Q from TMEM
            const auto issue_S = [&](int m) {
                const uint64_t b0 = bKk + step(m % NKR);
#pragma unroll
                for (int kk = 0; kk < 4 * DCH; ++kk) {
                    if (kk >= nk) break;
                    const uint64_t off = uint64_t(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
                    mma_ts(tmem, tmem + 448 + kk * 8, b0 + off, idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(s_full));
            };
            const auto issue_dP = [&](int m) {
                bwd_mma_rows<DCH>(tmem + 128, adO, bVk + step(m % NVR), idS, nk);
                mma_commit(smem_u32(dp_full));
                mma_commit(smem_u32(&v_empty[m % NVR]));
            };
            bool ok = mbar_wait(smem_u32(q_full), 0, p.timeout_ns, abort_flag);
            if (ok) ok = mbar_wait(smem_u32(q_tmem), 0, p.timeout_ns, abort_flag);
            if (ok) ok = kfull(0);
            if (ok) {
                tc_fence_after();
                issue_S(0);
                ok = vfull(0);
            }
            if (ok) {
                tc_fence_after();
                issue_dP(0);
            }
            for (int n = 0; n < n_kv && ok; ++n) {
                const bool more = n + 1 < n_kv;
                ok = mbar_wait(smem_u32(s_read), n & 1, p.timeout_ns, abort_flag);
                if (!ok) break;
                if (more) {
                    ok = kfull(n + 1);
                    if (!ok) break;
                    tc_fence_after();
                    issue_S(n + 1);
                }
                ok = mbar_wait(smem_u32(dp_read), n & 1, p.timeout_ns, abort_flag);
                if (!ok) break;
                if (more) {
                    ok = vfull(n + 1);
                    if (!ok) break;
                    tc_fence_after();
                    issue_dP(n + 1);
                }
                ok = mbar_wait(smem_u32(ds_ready), n & 1, p.timeout_ns, abort_flag);
                if (!ok) break;
                tc_fence_after();
                // dS columns 0-127 are TMEM columns 384-447 in order
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + 256, tmem + 384 + kk * 8, bKm + step(n % NKR) + uint64_t((kk * 2048) >> 4),
                           idA, (n > 0 || kk > 0) ? 1u : 0u);
                mma_commit(smem_u32(ds_free));
                mma_commit(smem_u32(&k_empty[n % NKR]));
            }
            mma_commit(smem_u32(acc_done));
            mbar_wait(smem_u32(acc_done), 0, p.timeout_ns, nullptr);
        }
    } else if (warp >= 4) {
        // ================================================= elementwise (one query row per thread)
        const int wq = warp & 3;
        const int half = (warp - 4) >> 2;         // key columns 64*half .. 64*half + 63
        const int row = wq * 32 + lane;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + 64 * half;
        const uint32_t tdP = tmem + lane_base + 128 + 64 * half;
        const uint32_t tdS = tmem + lane_base + 384 + 32 * half;
        const int i = qt * 128 + row;
        const size_t ro = size_t(bh) * p.Tpad + size_t(i);
        const float nl = p.nl[ro];
        const float dd = p.dd[ro];
        const float c2 = p.scale_log2;
        // Q row into TMEM (the A operand of S = Q K^T): this half's 64 columns
        // are one 128-byte row of its swizzled chunk
        bool ok = mbar_wait(smem_u32(q_full), 0, p.timeout_ns, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            const uint32_t qrow = sQ + uint32_t(half) * kChunkBytes + uint32_t(row >> 3) * 1024 + uint32_t(row & 7) * 128;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w[4 * u]), "=r"(w[4 * u + 1]), "=r"(w[4 * u + 2]), "=r"(w[4 * u + 3])
                                 : "r"(qrow + (uint32_t((4 * g + u) ^ (row & 7)) << 4)));
                tmem_st16(tmem + lane_base + 448 + 32 * half + 16 * g, w);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(q_tmem));
        }
        for (int n = 0; n < n_kv && ok; ++n) {
            ok = mbar_wait(smem_u32(s_full), n & 1, p.timeout_ns, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[2][32];
            tmem_ld32(tS + 0, r[0]);
            tmem_ld32(tS + 32, r[1]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(s_read));
            // key j = 128 n + c is visible when j < T and (not causal or j <= i);
            // `last` is counted from this half's first column
            const int nt = n_first + n;
            int last = 127;
            if (nt * 128 + 127 >= p.T) last = p.T - 1 - nt * 128;
            if (p.causal && nt == qt) last = min(last, row);
            last -= 64 * half;
            // with a window keys at or below i - w are not seen either
            const int first = WINDOW ? i - p.window + 1 - nt * 128 - 64 * half : -1;
            const float2 c2v = make_float2(c2, c2);
            const float2 nlv = make_float2(nl, nl);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float2 x = __ffma2_rn(make_float2(__uint_as_float(r[ch][2 * e]),
                                                      __uint_as_float(r[ch][2 * e + 1])),
                                          c2v, nlv);
                    if (32 * ch + 2 * e > last) x.x = -INFINITY;
                    if (32 * ch + 2 * e + 1 > last) x.y = -INFINITY;
                    if (WINDOW && 32 * ch + 2 * e < first) x.x = -INFINITY;
                    if (WINDOW && 32 * ch + 2 * e + 1 < first) x.y = -INFINITY;
                    r[ch][2 * e] = __float_as_uint(ex2(x.x));
                    r[ch][2 * e + 1] = __float_as_uint(ex2(x.y));
                }
            ok = mbar_wait(smem_u32(dp_full), n & 1, p.timeout_ns, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const float2 ndd = make_float2(-dd, -dd);
            // dS = P (dP - D) in place of P, then dP's columns are free
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t g[32];
                tmem_ld32(tdP + 32 * ch, g);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 pp = make_float2(__uint_as_float(r[ch][2 * e]), __uint_as_float(r[ch][2 * e + 1]));
                    const float2 t = __fadd2_rn(make_float2(__uint_as_float(g[2 * e]), __uint_as_float(g[2 * e + 1])), ndd);
                    const float2 ds = __fmul2_rn(pp, t);
                    r[ch][2 * e] = __float_as_uint(ds.x);
                    r[ch][2 * e + 1] = __float_as_uint(ds.y);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(dp_read));
            // dQ(n-1) must have read the previous dS
            if (n > 0) ok = mbar_wait(smem_u32(ds_free), (n - 1) & 1, p.timeout_ns, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack2<T>(__uint_as_float(r[ch][2 * e]), __uint_as_float(r[ch][2 * e + 1]));
                tmem_st16(tdS + 16 * ch, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(ds_ready));
        }
        if (ok) ok = mbar_wait(smem_u32(acc_done), 0, p.timeout_ns, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const bool valid = i < p.T;
            const size_t orow = (size_t(bh) * p.T + (valid ? i : 0)) * p.d;
            // the two halves store alternate 16-column pieces of the row
            bwd_store_row<T>(tmem + lane_base + 256, p.d, p.scale, static_cast<T*>(p.dq) + orow, valid,
                             16 * half, 32);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace b200attn
