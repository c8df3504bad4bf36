// Fused causal prefill attention on the 5th-generation tensor cores.
//
// Q.K^T and P.V are real dense contractions, so both run as tcgen05 MMAs
// with fp32 accumulators in tensor memory (TMEM); the softmax between them is
// the online form ("Causal Multi-Head Self-Attention", Two exact
// full-sequence algorithms: running row maximum and exponential sum, updated
// as each key tile arrives) with exp2 and the scale folded into the exponent.
//
// CTA work unit = two "slots", each a 128-query-row tile of one head:
//   * group size G even: two query heads of the same K/V head, same rows, so
//     every K/V tile loaded to shared memory feeds both heads ("Grouped-Query
//     Attention" §5.1 without the repeat_interleave copy);
//   * G odd (MHA, G = 1): one head, two consecutive 128-row tiles.
// Units are ordered heaviest first (longest causal row range first) and dealt
// to persistent CTAs (one per SM) in a snake order; barrier phases keep
// counting across a CTA's units, so the next unit's Q and first K/V copies
// and its first Q.K^T overlap the current unit's last tiles and epilogue.
// When the last pass would leave most CTAs idle, its units are cut into
// `split` pieces along the key tiles (the split-KV idea of the decode kernel
// applied to a prefill tail): each piece writes its O / l and log2-sum-exp
// in fp32 to a workspace and prefill_merge_kernel combines them.
//
// Warp roles (12 warps):
//   warp 0      TMA producer: per unit the Q tiles (once the previous unit's
//               last Q.K^T has read them), then K_n, V_n into a ring of NST
//               128-key stages (128-byte swizzle, zero fill past the end);
//   warp 1      TMEM owner (allocates all 512 columns) and single-thread MMA
//               issuer: S_s = Q_s K_n^T (SS MMA, M=N=128), O_s += P_s V_n
//               (TS MMA: P read straight from TMEM, N = d);
//   warp 2      (paged caches only) zeroes the V rows of a sequence's last
//               page past its length before P.V reads the stage;
//   warps 4-7   softmax for slot 0, warps 8-11 softmax for slot 1: one
//               thread per query row (TMEM lane), 128 scores in registers.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512);
// P_s (16-bit, two per column) overwrites the first 64 columns of S_s.
// Order per key tile n (two slots ping-pong so one slot's softmax overlaps
// the other slot's MMAs):  wait P_0(n) -> O_0 += P_0 V_n -> S_0(n+1);
//                          wait P_1(n) -> O_1 += P_1 V_n -> S_1(n+1).
// Key tiles entirely above the diagonal are never loaded; only tiles that
// straddle the diagonal (or the end of the keys) are masked.
//
// The running maximum is updated lazily: it is only raised (and O rescaled in
// TMEM) when the tile maximum exceeds it by more than 2^8 in the exp2 domain;
// otherwise the stale maximum keeps every P below 256, exact after the final
// division by l.
//
// The code of warpgroup 0 (producer, MMA issuer, paged-tail warp) holds no
// 64-bit integer division or remainder by a run-time value.  Twice, such a
// division added to that code (once executed per unit, once in a branch that
// never ran for the failing calls) made the windowed MHA prefill wrong at d =
// 128 with a window of about one key tile: the scores of a unit's second
// slot, whose window starts one key tile after the first slot's, came out
// wrong for that first tile, deterministically, while the same arithmetic in
// 32-bit form gave correct results.  The mechanism was not found.
#pragma once

#include "ptx.cuh"

namespace b200attn {

struct PrefillParams {
    void* o;
    float* lse;
    int B, H, Hkv, G, Tq;
    int64_t S;           // keys 0..S-1 exist
    int64_t start_pos;   // absolute position of query row 0
    int d;
    int causal;
    int64_t window;      // local window w: the row at p sees p - w < j <= p (0: none)
    int pair_mode;       // 0: two heads share a row tile; 1: one head, two row tiles
    int n_qb;            // ceil(Tq / 128)
    int units_per_level;
    int n_levels;        // units = units_per_level * n_levels, heaviest level first
    int group;           // units of a level taken together (grouped_order)
    // work items: units [0, n_whole) whole, then every later unit as `split`
    // pieces over its key tiles (ws_o / ws_lse: a piece's fp32 O / l and
    // m + log2 l per row, [piece][slot][128 rows][d] and [piece][slot][128])
    int n_whole, split;
    float* ws_o;
    float* ws_lse;
    float scale_log2;    // |scale| * log2(e) (1 when scale = 0)
    int score_mode;      // 0: scale > 0; 1: scale < 0 (scores negated); 2: scale = 0 (scores zeroed)
    uint64_t timeout_ns;
    uint32_t test_flags;  // kTestSkipLoads: issue no K/V copies (timeout-path tests)
    // paged K/V (the PAGED kernel): pools [num_pages, Hkv, 2^page_shift, d];
    // key j of sequence b is row j % P of page page_table[b * max_pages + j / P];
    // sequence b holds kv_lens[b] keys, its Tq new queries being the last ones
    const int32_t* page_table;
    const int32_t* kv_lens;
    int64_t max_pages, num_pages, max_kv_len;
    int page_shift;
};

constexpr int kPfThreads = 384;  // 12 warps
// Register split: warpgroup 0 (producer, issuer, two idle warps) gives
// registers up, the two softmax warpgroups (a row of 128 scores per thread)
// take them.  Needs launch registers x 384 >= 128 x low + 256 x high.
constexpr int kPfRegsLow = 120, kPfRegsHigh = 192;
constexpr uint32_t kChunkBytes = 128 * 128;  // 128 rows x 64 16-bit columns (one swizzle atom column)
constexpr float kRescaleThreshold = 8.0f;    // log2 units
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Columns past `last` of a 32-column chunk of scores (fp32 bits) become -inf.
__device__ __forceinline__ void mask_chunk(uint32_t (&r)[32], int last) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
        if (c > last) r[c] = 0xff800000u;  // -inf
}

// Columns before `first` of a 32-column chunk become -inf (a window's edge).
__device__ __forceinline__ void mask_chunk_below(uint32_t (&r)[32], int first) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
        if (c < first) r[c] = 0xff800000u;  // -inf
}

// Maximum of a 32-column chunk (fp32 bits): four independent max3 chains.
__device__ __forceinline__ float chunk_max(const uint32_t (&r)[32]) {
    float m[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) m[a] = fmax3(__uint_as_float(r[a]), __uint_as_float(r[a + 4]),
                                             __uint_as_float(r[a + 8]));
#pragma unroll
    for (int c = 12; c < 28; c += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a)
            m[a] = fmax3(m[a], __uint_as_float(r[c + a]), __uint_as_float(r[c + a + 4]));
#pragma unroll
    for (int a = 0; a < 4; ++a) m[a] = fmaxf(m[a], __uint_as_float(r[28 + a]));
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// P = 2^(s*c - m) for a 32-column chunk: the fp32 values replace the scores
// in r, the 16-bit pairs go to TMEM at `taddr` (16 columns).
template <typename T>
__device__ __forceinline__ void exp_chunk(uint32_t (&r)[32], float2 c2v, float2 negm, uint32_t taddr) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                                    c2v, negm);
        const float p0 = ex2(x.x), p1 = ex2(x.y);
        r[2 * i] = __float_as_uint(p0);
        r[2 * i + 1] = __float_as_uint(p1);
        pk[i] = pack2<T>(p0, p1);
    }
    tmem_st16(taddr, pk);
}

// Sum of a 32-column chunk of fp32 values (bits), four packed partial sums.
__device__ __forceinline__ float chunk_sum(const uint32_t (&r)[32]) {
    float2 acc[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[a] = make_float2(__uint_as_float(r[2 * a]), __uint_as_float(r[2 * a + 1]));
#pragma unroll
    for (int i = 8; i < 32; i += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a)
            acc[a] = __fadd2_rn(acc[a], make_float2(__uint_as_float(r[i + 2 * a]), __uint_as_float(r[i + 2 * a + 1])));
    const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
    const float2 t = __fadd2_rn(s01, s23);
    return t.x + t.y;
}

template <int DCH> struct PrefillRing { static constexpr int NST = DCH == 2 ? 4 : 8; };

template <int DCH>
constexpr size_t prefill_smem_bytes() {
    return 1024 + size_t(2 + PrefillRing<DCH>::NST) * DCH * kChunkBytes + 512;
}

// A slot's key tiles: it needs tiles [n_lo, n_kv); tiles in [n_full_lo,
// n_full) are visible to every row of it, the others are masked.
struct SlotInfo {
    int h, q0, n_lo, n_kv, n_full_lo, n_full;
    int64_t S, start;   // keys of the slot's sequence, position of its query row 0
};

template <bool WINDOW>
__device__ __forceinline__ SlotInfo prefill_slot(const PrefillParams& p, int h, int qb, int64_t S,
                                                 int64_t start) {
    SlotInfo s;
    s.h = h;
    s.q0 = qb * 128;
    s.S = S;
    s.start = start;
    if (s.q0 >= p.Tq) {
        s.n_lo = s.n_kv = s.n_full_lo = s.n_full = 0;
        return s;
    }
    const int64_t qlast = min64(s.q0 + 127, p.Tq - 1);
    const int64_t kv_end = p.causal ? min64(S, start + qlast + 1) : S;
    s.n_kv = int((kv_end + 127) / 128);
    const int64_t full_c = p.causal ? (start + s.q0 + 1) / 128 : (S / 128);
    s.n_full = int(min64(full_c, S / 128));
    s.n_lo = s.n_full_lo = 0;
    if (WINDOW) {
        const int64_t first = max64(0, start + s.q0 - p.window + 1);   // lowest key seen
        const int64_t all_lo = max64(0, start + qlast - p.window + 1);  // every row sees from here
        s.n_lo = int(first / 128);
        s.n_full_lo = int((all_lo + 127) / 128);
    }
    return s;
}

// S_s = Q_s K^T over d/16 k-steps.  Descriptors advance by adding (byte
// offset >> 4) to their start-address field; the offsets are compile-time
// constants, so each MMA issues without a descriptor being rebuilt (an MMA
// stream whose descriptors are rebuilt per instruction issues more slowly than
// the tensor pipe retires it).
template <int DCH>
__device__ __forceinline__ void issue_S(uint64_t dQ0, uint64_t dK0, uint32_t tmem, uint32_t idS,
                                        int nk, int s, int st) {
    constexpr uint32_t kStageStep = (DCH * kChunkBytes) >> 4;
    const uint64_t a0 = dQ0 + uint64_t(uint32_t(s) * kStageStep);
    const uint64_t b0 = dK0 + uint64_t(uint32_t(st) * kStageStep);
    const uint32_t dS = tmem + s * 128;
#pragma unroll
    for (int kk = 0; kk < 4 * DCH; ++kk) {
        if (kk >= nk) break;
        const uint64_t off = uint64_t(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
        mma_ss(dS, a0 + off, b0 + off, idS, kk > 0 ? 1u : 0u);
    }
}

// O_s (+)= P_s V for keys 16*K0 .. 16*K0 + 63 (P read from TMEM).
template <int K0, int DCH>
__device__ __forceinline__ void issue_PV(uint64_t dV0, uint32_t tmem, uint32_t idO, int s, int st,
                                         bool accumulate) {
    constexpr uint32_t kStageStep = (DCH * kChunkBytes) >> 4;
    const uint64_t b0 = dV0 + uint64_t(uint32_t(st) * kStageStep);
    const uint32_t dO = tmem + 256 + s * 128;
    const uint32_t aP = tmem + s * 128;
#pragma unroll
    for (int kk = K0; kk < K0 + 4; ++kk)
        mma_ts(dO, aP + kk * 8, b0 + uint64_t((kk * 2048) >> 4), idO,
               (accumulate || kk > 0) ? 1u : 0u);
}

// Work order with L2 locality.  The units are `per_level` items (batch
// entries and heads) times `n_levels` levels of decreasing work.  Walking
// level by level puts one tile of every item in flight at once, and at
// several GB of K/V the tiles a CTA reuses are gone from L2 by then; so the
// items are taken in groups of `group` consecutive ones whose tiles fit in L2
// together, each group heaviest level first.  Unit -> (level, item).
__host__ __device__ __forceinline__ void grouped_order(int unit, int per_level, int n_levels, int group,
                                                       int& level, int& item) {
    // 32-bit throughout: the planners keep every unit count below 2^31
    const int full = per_level / group;             // whole groups
    const int span = group * n_levels;
    if (unit < full * span) {
        const int g = unit / span, r = unit % span;
        level = r / group;
        item = g * group + r % group;
    } else {
        const int last = per_level - full * group;  // > 0 here
        const int r = unit - full * span;
        level = r / last;
        item = full * group + r % last;
    }
}

// The unit of work a CTA does at pass `unit`: its batch entry, K/V head and
// two slots (heaviest first within a group of K/V heads: the longest causal
// row range first).
template <bool WINDOW, bool PAGED>
__device__ __forceinline__ void prefill_unit(const PrefillParams& p, int unit, int& b, int& kvh,
                                             SlotInfo (&slot)[2]) {
    int level, rem;
    grouped_order(unit, p.units_per_level, p.n_levels, p.group, level, rem);
    int h0, h1, qb0, qb1;
    if (p.pair_mode == 0) {
        const int half = p.G / 2;
        b = rem / (p.Hkv * half);
        const int r2 = rem % (p.Hkv * half);
        kvh = r2 / half;
        h0 = kvh * p.G + 2 * (r2 % half);
        h1 = h0 + 1;
        qb0 = qb1 = p.n_qb - 1 - level;
    } else {
        const int qbp = p.n_levels - 1 - level;
        b = rem / p.H;
        h0 = h1 = rem % p.H;
        kvh = h0 / p.G;
        qb0 = 2 * qbp;
        qb1 = qb0 + 1;
    }
    int64_t S = p.S, start = p.start_pos;
    if (PAGED) {
        // a length outside [Tq, max_kv_len] is reported and clamped
        int64_t L = p.kv_lens[b];
        if (L < p.Tq || L > p.max_kv_len) {
            atomicCAS(&g_device_status, 0u, kStatusBadIndex);
            L = max64(int64_t(p.Tq), min64(L, p.max_kv_len));
        }
        S = L;
        start = L - p.Tq;
    }
    slot[0] = prefill_slot<WINDOW>(p, h0, qb0, S, start);
    slot[1] = prefill_slot<WINDOW>(p, h1, qb1, S, start);
}

// Work items: unit `item` while item < n_whole, then piece
// (item - n_whole) % split of unit n_whole + (item - n_whole) / split.  A
// piece keeps the key tiles [lo, hi) of its part of the unit's range; a slot
// left with none is empty (n_kv = 0).  Returns the piece index, or -1 for a
// whole unit.
__host__ __device__ __forceinline__ int prefill_items(const PrefillParams& p) {
    return p.n_whole + (p.units_per_level * p.n_levels - p.n_whole) * p.split;
}

template <bool WINDOW, bool PAGED, bool SPLIT>
__device__ __forceinline__ int prefill_item(const PrefillParams& p, int item, int& b, int& kvh,
                                            SlotInfo (&slot)[2]) {
    if (!SPLIT || item < p.n_whole) {
        prefill_unit<WINDOW, PAGED>(p, item, b, kvh, slot);
        return -1;
    }
    const int piece = item - p.n_whole;
    const int part = piece % p.split;
    prefill_unit<WINDOW, PAGED>(p, p.n_whole + piece / p.split, b, kvh, slot);
    int n0 = 0x7fffffff, n1 = 0;
#pragma unroll
    for (int s = 0; s < 2; ++s)
        if (slot[s].n_kv > 0) {
            n0 = min(n0, slot[s].n_lo);
            n1 = max(n1, slot[s].n_kv);
        }
    if (n1 == 0) return piece;
    // 32-bit: a unit spans fewer than 2^26 key tiles (S * d * 2 < 2^40 with
    // d >= 64, checked on the host), times part + 1 <= 4.  The warps of
    // warpgroup 0 run no 64-bit division by a run-time value (see the note
    // at the top of the kernel).
    const int lo = n0 + (n1 - n0) * part / p.split;
    const int hi = n0 + (n1 - n0) * (part + 1) / p.split;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        if (slot[s].n_kv == 0) continue;
        slot[s].n_lo = max(slot[s].n_lo, lo);
        slot[s].n_kv = min(slot[s].n_kv, hi);
        if (slot[s].n_lo >= slot[s].n_kv) slot[s].n_lo = slot[s].n_kv = 0;
    }
    return piece;
}

// K or V tile n of sequence b, head kvh, from a paged pool: one TMA copy per
// page the tile spans (min(P, 128) rows each).  Copies that start at or past
// the sequence's end, and pages whose id is out of range (reported), are read
// at an out-of-range coordinate, which TMA fills with zeros while still
// counting the bytes.  The copy that holds the sequence's last rows brings the
// rest of its page too; those rows of a V tile are zeroed in shared memory by
// the tail warp before P.V reads them.
template <int DCH>
__device__ __forceinline__ void load_kv_paged(const PrefillParams& p, uint32_t dst, const CUtensorMap* map,
                                              uint32_t bar, int n, int b, int kvh, int64_t L) {
    const int rows = min(1 << p.page_shift, 128);
    for (int sub = 0; sub < 128 / rows; ++sub) {
        const int64_t tok = int64_t(n) * 128 + int64_t(sub) * rows;
        int64_t z = p.num_pages * p.Hkv;   // past the pools: zero fill
        int y = 0;
        if (tok < L) {
            const int32_t phys = p.page_table[int64_t(b) * p.max_pages + (tok >> p.page_shift)];
            if (phys < 0 || phys >= p.num_pages) {
                atomicCAS(&g_device_status, 0u, kStatusBadIndex);
            } else {
                z = int64_t(phys) * p.Hkv + kvh;
                y = int(tok & ((int64_t(1) << p.page_shift) - 1));
            }
        }
        for (int c = 0; c < DCH; ++c)
            tma_load_3d(dst + c * kChunkBytes + uint32_t(sub * rows) * 128u, map, bar, c * 64, y, int32_t(z));
    }
}

// Unit dealt to this CTA at pass k: a snake over the grid (CTA c takes
// units c, 2G - 1 - c, 2G + c, ...), so heavy and light units even out.
__device__ __forceinline__ int prefill_pass_unit(int k) {
    return (k & 1) == 0 ? k * int(gridDim.x) + int(blockIdx.x)
                        : (k + 1) * int(gridDim.x) - 1 - int(blockIdx.x);
}

// SPLIT: the launch has pieces (n_whole < units); the kernels of launches
// without them carry no piece code (it cost the BitNet-3B prefill 4 %).
template <typename T, int DCH, bool WINDOW, bool PAGED, bool SPLIT>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_tcgen05_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
    constexpr int NST = PrefillRing<DCH>::NST;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char* base_ptr = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t sQ = base;                                      // [2][DCH] chunks
    const uint32_t sRing = base + 2 * DCH * kChunkBytes;           // [NST][DCH] chunks
    uint64_t* bars = reinterpret_cast<uint64_t*>(base_ptr + (2 + NST) * DCH * kChunkBytes);
    uint64_t* q_full = bars;            // 2
    uint64_t* q_empty = bars + 2;       // 2
    uint64_t* kv_full = bars + 4;       // NST
    uint64_t* kv_empty = kv_full + NST; // NST
    uint64_t* s_full = kv_empty + NST;  // 2
    uint64_t* p_ready = s_full + 2;     // [slot][half]: 4
    uint64_t* o_done = p_ready + 4;     // 2
    uint64_t* drain = o_done + 2;       // 1
    uint64_t* kv_ready = drain + 1;     // NST (PAGED: V stages with their tail rows zeroed)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(kv_ready + NST);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_items = prefill_items(p);

    // Persistent CTAs work through their units as one pipeline: every barrier
    // keeps counting phases across units (each role tracks its own counts),
    // so the producer loads the next unit's Q and first K/V tiles while this
    // unit's last tiles and epilogue run, and the issuer starts the next
    // unit's first Q.K^T as soon as they land.
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&q_full[s]), 1);
            mbar_init(smem_u32(&q_empty[s]), 1);
            mbar_init(smem_u32(&s_full[s]), 1);
            mbar_init(smem_u32(&p_ready[2 * s]), 4);      // one arrive per softmax warp
            mbar_init(smem_u32(&p_ready[2 * s + 1]), 4);
            mbar_init(smem_u32(&o_done[s]), 1);
        }
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&kv_full[i]), 1);
            mbar_init(smem_u32(&kv_empty[i]), 1);
            mbar_init(smem_u32(&kv_ready[i]), 1);
        }
        mbar_init(smem_u32(drain), 1);
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
    if (warp < 4) {
        reg_dealloc<kPfRegsLow>();
        if (warp == 0) {
            // ================================================= TMA producer
            if (lane == 0) {
                tma_prefetch_desc(&tmQ);
                tma_prefetch_desc(&tmK);
                tma_prefetch_desc(&tmV);
                uint32_t qcount[2] = {0, 0};   // Q loads per slot so far
                int64_t li = 0;                // K/V loads so far (ring position)
                bool ok = true;
                for (int pass = 0; ok; ++pass) {
                    const int unit = prefill_pass_unit(pass);
                    if (unit >= n_items) break;
                    int b, kvh;
                    SlotInfo slot[2];
                    prefill_item<WINDOW, PAGED, SPLIT>(p, unit, b, kvh, slot);
                    const int nmax = max(slot[0].n_kv, slot[1].n_kv);
                    const int nmin = slot[0].n_kv == 0 ? slot[1].n_lo
                                     : slot[1].n_kv == 0 ? slot[0].n_lo : min(slot[0].n_lo, slot[1].n_lo);
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        if (slot[s].n_kv == 0) continue;
                        // the previous unit's Q.K^T MMAs of this slot are done with Q
                        if (qcount[s] > 0 &&
                            !mbar_wait(smem_u32(&q_empty[s]), (qcount[s] - 1) & 1, p.timeout_ns, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t bar = smem_u32(&q_full[s]);
                        mbar_expect_tx(bar, DCH * kChunkBytes);
                        for (int c = 0; c < DCH; ++c)
                            tma_load_3d(sQ + (s * DCH + c) * kChunkBytes, &tmQ, bar, c * 64, slot[s].q0,
                                        b * p.H + slot[s].h);
                        ++qcount[s];
                    }
                    const int zkv = b * p.Hkv + kvh;
                    const int n_loads = (p.test_flags & kTestSkipLoads) ? 0 : 2 * (nmax - nmin);
                    for (int i = 0; i < n_loads && ok; ++i, ++li) {
                        const int st = int(li % NST);
                        if (!mbar_wait(smem_u32(&kv_empty[st]), uint32_t((li / NST) & 1) ^ 1, p.timeout_ns,
                                       abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t bar = smem_u32(&kv_full[st]);
                        mbar_expect_tx(bar, DCH * kChunkBytes);
                        const CUtensorMap* map = (i & 1) ? &tmV : &tmK;
                        if (PAGED)
                            load_kv_paged<DCH>(p, sRing + st * DCH * kChunkBytes, map, bar, nmin + (i >> 1), b,
                                               kvh, slot[0].S);
                        else
                            for (int c = 0; c < DCH; ++c)
                                tma_load_3d(sRing + (st * DCH + c) * kChunkBytes, map, bar, c * 64,
                                            (nmin + (i >> 1)) * 128, zkv);
                    }
                }
                // no copy may still be landing in shared memory when the CTA exits
                for (int64_t i = li - 1; i >= 0 && i >= li - NST; --i)
                    mbar_wait(smem_u32(&kv_full[i % NST]), uint32_t((i / NST) & 1), p.timeout_ns, nullptr);
                for (int s = 0; s < 2; ++s)
                    if (qcount[s] > 0)
                        mbar_wait(smem_u32(&q_full[s]), (qcount[s] - 1) & 1, p.timeout_ns, nullptr);
            }
        } else if (warp == 1) {
            // ================================================= MMA issuer
            if (lane == 0) {
                const uint32_t idS = idesc_f16(kBF16, 128, 128, false);
                const uint32_t idO = idesc_f16(kBF16, 128, p.d, true);
                const int nk = p.d / 16;
                const uint64_t dQ0 = smem_desc_sw128(sQ, 16, 1024);
                const uint64_t dK0 = smem_desc_sw128(sRing, 16, 1024);
                const uint64_t dV0 = smem_desc_sw128(sRing, kChunkBytes, 1024);
                uint32_t qcount[2] = {0, 0};   // units started per slot
                uint32_t pcount[2] = {0, 0};   // tiles whose P was consumed, per slot
                int64_t li = 0;                // K/V loads consumed (ring position)
                bool ok = true;
                for (int pass = 0; ok; ++pass) {
                    const int unit = prefill_pass_unit(pass);
                    if (unit >= n_items) break;
                    int b, kvh;
                    SlotInfo slot[2];
                    prefill_item<WINDOW, PAGED, SPLIT>(p, unit, b, kvh, slot);
                    const int nmax = max(slot[0].n_kv, slot[1].n_kv);
                    const int nmin = slot[0].n_kv == 0 ? slot[1].n_lo
                                     : slot[1].n_kv == 0 ? slot[0].n_lo : min(slot[0].n_lo, slot[1].n_lo);
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        if (slot[s].n_kv == 0 || !ok) continue;
                        ok = mbar_wait(smem_u32(&q_full[s]), qcount[s] & 1, p.timeout_ns, abort_flag);
                        ++qcount[s];
                    }
                    if (nmax == 0) continue;   // a piece with no key tiles: nothing was loaded
                    if (ok) ok = mbar_wait(smem_u32(&kv_full[li % NST]), uint32_t((li / NST) & 1), p.timeout_ns,
                                           abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    {
                        const int stK = int(li % NST);
#pragma unroll
                        for (int s = 0; s < 2; ++s) {
                            if (slot[s].n_kv == 0 || slot[s].n_lo != nmin) continue;
                            issue_S<DCH>(dQ0, dK0, tmem, idS, nk, s, stK);
                            mma_commit(smem_u32(&s_full[s]));
                            if (nmin + 1 == slot[s].n_kv) mma_commit(smem_u32(&q_empty[s]));
                        }
                        mma_commit(smem_u32(&kv_empty[stK]));
                        ++li;
                    }
                    for (int n = nmin; n < nmax && ok; ++n) {
                        const int64_t iV = li, iK = li + 1;
                        const int stV = int(iV % NST), stK = int(iK % NST);
                        const bool nextK = n + 1 < nmax;
                        ok = mbar_wait(smem_u32(PAGED ? &kv_ready[stV] : &kv_full[stV]), uint32_t((iV / NST) & 1),
                                       p.timeout_ns, abort_flag);
                        if (ok && nextK)
                            ok = mbar_wait(smem_u32(&kv_full[stK]), uint32_t((iK / NST) & 1), p.timeout_ns,
                                           abort_flag);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int s = 0; s < 2; ++s) {
                            // a slot whose window starts at tile n + 1 only gets its first S here
                            const bool first_next = WINDOW && n + 1 == slot[s].n_lo && n + 1 < slot[s].n_kv;
                            if (first_next) {
                                issue_S<DCH>(dQ0, dK0, tmem, idS, nk, s, stK);
                                mma_commit(smem_u32(&s_full[s]));
                                if (n + 2 == slot[s].n_kv) mma_commit(smem_u32(&q_empty[s]));
                            }
                            if (!ok || n < slot[s].n_lo || n >= slot[s].n_kv) continue;
                            const uint32_t par = pcount[s] & 1;
                            // P in two halves: the first 64 keys' MMAs start while the
                            // softmax is still producing the second half
                            if (!mbar_wait(smem_u32(&p_ready[2 * s]), par, p.timeout_ns, abort_flag)) {
                                ok = false;
                                continue;
                            }
                            tc_fence_after();
                            issue_PV<0, DCH>(dV0, tmem, idO, s, stV, n > slot[s].n_lo);
                            if (!mbar_wait(smem_u32(&p_ready[2 * s + 1]), par, p.timeout_ns, abort_flag)) {
                                ok = false;
                                continue;
                            }
                            tc_fence_after();
                            issue_PV<4, DCH>(dV0, tmem, idO, s, stV, true);
                            ++pcount[s];
                            if (n == slot[s].n_kv - 1) mma_commit(smem_u32(&o_done[s]));
                            if (n + 1 < slot[s].n_kv) {
                                issue_S<DCH>(dQ0, dK0, tmem, idS, nk, s, stK);
                                mma_commit(smem_u32(&s_full[s]));
                                if (n + 2 == slot[s].n_kv) mma_commit(smem_u32(&q_empty[s]));
                            }
                        }
                        if (!ok) break;
                        mma_commit(smem_u32(&kv_empty[stV]));
                        ++li;
                        if (nextK) {
                            mma_commit(smem_u32(&kv_empty[stK]));
                            ++li;
                        }
                    }
                }
                // every MMA issued must finish before TMEM is released
                mma_commit(smem_u32(drain));
                mbar_wait(smem_u32(drain), 0, p.timeout_ns, nullptr);
            }
        } else if (PAGED && warp == 2) {
            // ================================================= paged V tails
            // A copy brings whole page rows, so the rows of a sequence's last
            // page past its length L arrive with it.  They enter P.V with
            // weight 0, and 0 * NaN (or inf) is NaN: the result must not
            // depend on what unused page rows hold, so they are zeroed here,
            // in shared memory, before any MMA reads the V stage.  Every V
            // stage passes through this warp (kv_full -> kv_ready).  K needs
            // nothing: the scores of keys at or past L are overwritten by the
            // mask.  Loads alternate K, V and a unit issues an even number of
            // them, so with an even ring every use of a V stage is a V load
            // and kv_ready's phases follow kv_full's.
            static_assert(NST % 2 == 0, "V loads must keep to their own stages");
            const int copy_shift = min(p.page_shift, 7);   // a copy brings min(P, 128) rows
            int64_t li = 0;
            bool ok = true;
            for (int pass = 0; ok; ++pass) {
                const int unit = prefill_pass_unit(pass);
                if (unit >= n_items) break;
                int b, kvh;
                SlotInfo slot[2];
                prefill_item<WINDOW, PAGED, SPLIT>(p, unit, b, kvh, slot);
                const int nmax = max(slot[0].n_kv, slot[1].n_kv);
                const int nmin = slot[0].n_kv == 0 ? slot[1].n_lo
                                 : slot[1].n_kv == 0 ? slot[0].n_lo : min(slot[0].n_lo, slot[1].n_lo);
                const int n_loads = (p.test_flags & kTestSkipLoads) ? 0 : 2 * (nmax - nmin);
                const int64_t L = slot[0].S;
                // rows [L, end of the copy holding row L - 1) came from the pool
                const int64_t tail_end = ((L + (int64_t(1) << copy_shift) - 1) >> copy_shift) << copy_shift;
                for (int i = 0; i < n_loads && ok; ++i, ++li) {
                    if ((i & 1) == 0) continue;
                    const int st = int(li % NST);
                    ok = mbar_wait(smem_u32(&kv_full[st]), uint32_t((li / NST) & 1), p.timeout_ns, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    const int64_t t0 = int64_t(nmin + (i >> 1)) * 128;
                    const int r0 = int(max64(0, min64(128, L - t0)));
                    const int r1 = int(max64(0, min64(128, tail_end - t0)));
                    if (r1 > r0) {
                        // whole 128-byte rows: the swizzle only permutes 16-byte
                        // pieces within a row
                        const uint32_t dst = sRing + uint32_t(st * DCH) * kChunkBytes + uint32_t(r0) * 128u;
                        const int per_chunk = (r1 - r0) * 8;
                        for (int x = lane; x < DCH * per_chunk; x += 32) {
                            const int c = x / per_chunk;
                            const uint32_t a = dst + uint32_t(c) * kChunkBytes + uint32_t(x - c * per_chunk) * 16u;
                            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&kv_ready[st]));
                }
            }
        }
    } else {
        reg_alloc<kPfRegsHigh>();
        // ================================================= softmax + epilogue
        // warps 4-7: slot 0, warps 8-11: slot 1; one thread per row (TMEM lane).
        const int s = (warp - 4) >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t tS = tmem + (uint32_t(wq * 32) << 16) + s * 128;
        const uint32_t tO = tmem + (uint32_t(wq * 32) << 16) + 256 + s * 128;
        const float c2 = p.scale_log2;
        uint32_t scount = 0, ocount = 0;   // S tiles and units consumed by this slot
        bool ok = true;
        for (int pass = 0; ok; ++pass) {
            const int unit = prefill_pass_unit(pass);
            if (unit >= n_items) break;
            int b, kvh;
            SlotInfo slot[2];
            const int piece = prefill_item<WINDOW, PAGED, SPLIT>(p, unit, b, kvh, slot);
            const SlotInfo sl = slot[s];
            if (sl.n_kv == 0) {
                // a piece's slot with no key tiles: its partial weighs nothing
                if (SPLIT && piece >= 0 && sl.q0 < p.Tq) p.ws_lse[(size_t(piece) * 2 + s) * 128 + row] = -INFINITY;
                continue;
            }
            const int64_t qpos = sl.start + sl.q0 + row;
            float m_run = -INFINITY, l = 0.f;
            bool first = true;   // the slot's first key tile of this item
            for (int n = sl.n_lo; n < sl.n_kv; ++n) {
                ok = mbar_wait(smem_u32(&s_full[s]), scount & 1, p.timeout_ns, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                ++scount;
                if (!ok) break;
                tc_fence_after();
                // All 128 scores of this row in registers (one wait: TMEM
                // loads are cheap next to the arithmetic that follows).
                uint32_t r0[32], r1[32], r2[32], r3[32];
                tmem_ld32(tS + 0, r0);
                tmem_ld32(tS + 32, r1);
                tmem_ld32(tS + 64, r2);
                tmem_ld32(tS + 96, r3);
                tmem_wait_ld();
                if (p.score_mode != 0) {
                    // scale < 0 is attention on -S with |scale|; scale = 0 weighs
                    // every visible key alike (the mask below still applies)
                    const uint32_t flip = p.score_mode == 1 ? 0x80000000u : 0u;
                    const uint32_t keep = p.score_mode == 1 ? 0xffffffffu : 0u;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        r0[e] = (r0[e] & keep) ^ flip;
                        r1[e] = (r1[e] & keep) ^ flip;
                        r2[e] = (r2[e] & keep) ^ flip;
                        r3[e] = (r3[e] & keep) ^ flip;
                    }
                }
                const bool masked = n >= sl.n_full || (WINDOW && n < sl.n_full_lo);
                if (masked) {
                    int64_t lim = p.causal ? qpos - int64_t(n) * 128 : 127;
                    lim = min64(lim, sl.S - 1 - int64_t(n) * 128);
                    const int li = int(max64(-1, min64(127, lim)));
                    mask_chunk(r0, li);
                    mask_chunk(r1, li - 32);
                    mask_chunk(r2, li - 64);
                    mask_chunk(r3, li - 96);
                    if (WINDOW) {
                        // keys at or below qpos - w are outside the window
                        const int lo = int(max64(0, min64(128, qpos - p.window + 1 - int64_t(n) * 128)));
                        mask_chunk_below(r0, lo);
                        mask_chunk_below(r1, lo - 32);
                        mask_chunk_below(r2, lo - 64);
                        mask_chunk_below(r3, lo - 96);
                    }
                }
                const float m_tile =
                    fmaxf(fmaxf(chunk_max(r0), chunk_max(r1)), fmaxf(chunk_max(r2), chunk_max(r3))) * c2;
                if (first) {
                    first = false;
                    m_run = m_tile;
                } else {
                    const bool need = m_tile - m_run > kRescaleThreshold;
                    if (__any_sync(0xffffffffu, need)) {
                        const float alpha = need ? ex2(m_run - m_tile) : 1.f;
                        if (need) {
                            l *= alpha;
                            m_run = m_tile;
                        }
                        // O_s is final for tile n-1 (its MMA completed before S_s(n))
                        for (int cc = 0; cc < p.d; cc += 16) {
                            uint32_t x[16];
                            tmem_ld16(tO + cc, x);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                x[e] = __float_as_uint(__uint_as_float(x[e]) * alpha);
                            tmem_st16(tO + cc, x);
                        }
                    }
                }
                // P = 2^(S*c - m) per 32-column chunk, packed to 16-bit pairs and
                // stored at once; the first 64 keys are released to the MMA
                // before the last 64 are computed.  r* then hold P in fp32.
                const float2 c2v = make_float2(c2, c2);
                // a row that has seen no key yet (a window starting in a later
                // tile, or a piece's range ending before the row's first key)
                // has m_run = -inf: its P must be 0, not NaN
                const float m_use = m_run == -INFINITY ? 0.f : m_run;
                const float2 negm = make_float2(-m_use, -m_use);
                exp_chunk<T>(r0, c2v, negm, tS + 0);
                exp_chunk<T>(r1, c2v, negm, tS + 16);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&p_ready[2 * s]));
                exp_chunk<T>(r2, c2v, negm, tS + 32);
                exp_chunk<T>(r3, c2v, negm, tS + 48);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&p_ready[2 * s + 1]));
                // row sum, off the MMA's critical path
                l += chunk_sum(r0) + chunk_sum(r1) + chunk_sum(r2) + chunk_sum(r3);
            }
            // ---- epilogue: O / l, rounded to the output type
            if (ok) ok = mbar_wait(smem_u32(&o_done[s]), ocount & 1, p.timeout_ns, abort_flag);
            ++ocount;
            ok = __all_sync(0xffffffffu, ok);
            const int item = prefill_pass_unit(pass);
            if (SPLIT && ok && item >= p.n_whole) {
                // a piece: O / l and m + log2 l in fp32 for the merge (a row
                // that saw no key of the piece has l = 0 and weighs nothing)
                tc_fence_after();
                const bool valid = sl.q0 + row < p.Tq;
                const size_t prow = (size_t(item - p.n_whole) * 2 + s) * 128 + row;
                float* wo = p.ws_o + prow * p.d;
                const float inv = l > 0.f ? 1.f / l : 0.f;
                for (int cc = 0; cc < p.d; cc += 16) {
                    uint32_t x[16];
                    tmem_ld16(tO + cc, x);
                    tmem_wait_ld();
                    if (valid) {
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *reinterpret_cast<float4*>(wo + cc + e) =
                                make_float4(__uint_as_float(x[e]) * inv, __uint_as_float(x[e + 1]) * inv,
                                            __uint_as_float(x[e + 2]) * inv, __uint_as_float(x[e + 3]) * inv);
                    }
                }
                if (valid) p.ws_lse[prow] = l > 0.f ? m_run + log2f(l) : -INFINITY;
            } else if (ok) {
                tc_fence_after();
                const bool valid = sl.q0 + row < p.Tq;
                const size_t orow = (size_t(b) * p.H + sl.h) * p.Tq + sl.q0 + row;
                T* optr = static_cast<T*>(p.o) + orow * p.d;
                const float inv = 1.f / l;
                for (int cc = 0; cc < p.d; cc += 16) {
                    uint32_t x[16];
                    tmem_ld16(tO + cc, x);
                    tmem_wait_ld();
                    uint4 w0, w1;
                    w0.x = pack2<T>(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv);
                    w0.y = pack2<T>(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv);
                    w0.z = pack2<T>(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv);
                    w0.w = pack2<T>(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv);
                    w1.x = pack2<T>(__uint_as_float(x[8]) * inv, __uint_as_float(x[9]) * inv);
                    w1.y = pack2<T>(__uint_as_float(x[10]) * inv, __uint_as_float(x[11]) * inv);
                    w1.z = pack2<T>(__uint_as_float(x[12]) * inv, __uint_as_float(x[13]) * inv);
                    w1.w = pack2<T>(__uint_as_float(x[14]) * inv, __uint_as_float(x[15]) * inv);
                    if (valid) {
                        reinterpret_cast<uint4*>(optr + cc)[0] = w0;
                        reinterpret_cast<uint4*>(optr + cc)[1] = w1;
                    }
                }
                if (valid && p.lse) p.lse[orow] = (m_run + log2f(l)) * 0.69314718055994531f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Merge of the pieces of the split units: per query row, the pieces' O_i and
// m_i + log2 l_i (log2 domain) combine as O = sum_i 2^(lse_i - M) O_i / W with
// M = max_i lse_i and W = sum_i 2^(lse_i - M); the row's log-sum-exp is
// (M + log2 W) ln 2.  One warp per row, four d-columns per lane, four rows
// per block.  (Measured against fewer, longer-lived warps that walk several
// rows each, or decode their unit once for 16 rows: both slower.)  Launched
// as a programmatic dependent of the prefill kernel: it waits for that grid's
// results before reading them.
constexpr int kMergeMaxSplit = 4;
constexpr int kMergeThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) prefill_merge_kernel(const PrefillParams p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int n_tail = p.units_per_level * p.n_levels - p.n_whole;
    const int64_t rid = int64_t(blockIdx.x) * (kMergeThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (rid >= int64_t(n_tail) * 256) return;
    const int ui = int(rid >> 8), s = int(rid >> 7) & 1, r = int(rid & 127);
    int b, kvh;
    SlotInfo slot[2];
    prefill_unit<false, false>(p, p.n_whole + ui, b, kvh, slot);
    const int h = s ? slot[1].h : slot[0].h, q0 = s ? slot[1].q0 : slot[0].q0;   // no indexed local array
    if (q0 + r >= p.Tq) return;
    // every piece's row is loaded at once (one memory round trip, not one for
    // the weights and another for the rows); a piece whose slot had no key
    // tile left its row unwritten, so its weight selects it away rather than
    // multiplying whatever the row holds
    const int c = lane * 4;
    float lse[kMergeMaxSplit];
    float4 x[kMergeMaxSplit];
#pragma unroll
    for (int i = 0; i < kMergeMaxSplit; ++i) {
        const size_t prow = ((size_t(ui) * p.split + i) * 2 + s) * 128 + r;
        lse[i] = i < p.split ? p.ws_lse[prow] : -INFINITY;
        x[i] = i < p.split && c < p.d ? *reinterpret_cast<const float4*>(p.ws_o + prow * p.d + c)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMergeMaxSplit; ++i) M = fmaxf(M, lse[i]);
    float W = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kMergeMaxSplit; ++i) {
        const bool live = lse[i] != -INFINITY;
        const float w = live ? ex2(lse[i] - M) : 0.f;
        W += w;
        acc.x += live ? w * x[i].x : 0.f;
        acc.y += live ? w * x[i].y : 0.f;
        acc.z += live ? w * x[i].z : 0.f;
        acc.w += live ? w * x[i].w : 0.f;
    }
    const float invW = W > 0.f ? 1.f / W : 0.f;
    const size_t orow = (size_t(b) * p.H + h) * p.Tq + q0 + r;
    if (c < p.d) {
        uint2 out;
        out.x = pack2<T>(acc.x * invW, acc.y * invW);
        out.y = pack2<T>(acc.z * invW, acc.w * invW);
        *reinterpret_cast<uint2*>(static_cast<T*>(p.o) + orow * p.d + c) = out;
    }
    if (lane == 0 && p.lse) p.lse[orow] = W > 0.f ? (M + log2f(W)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace b200attn
