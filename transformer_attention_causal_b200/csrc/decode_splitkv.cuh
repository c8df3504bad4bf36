// Split-KV cached-decode attention on CUDA cores: a few new query tokens per
// sequence against a long K/V history.  Used for d = 256 (head sizes 64 and
// 128 run on the warp-level MMA kernel of decode_mma.cuh, which shares this
// file's parameters, span helper and combine kernel).  HBM-bound: every call streams the visible
// history once ("Multi-query attention, annotated" §2.4.1: incremental
// attention rereads the whole cache at about one multiply-add per number
// read), so the kernel is built around keeping HBM busy, not around FLOPs.
//
// Work unit: (b, kv head, key split).  All G = H / Hkv query heads of a K/V
// head, times Tnew new tokens, form R rows that share every K/V row read
// ("Grouped-Query Attention" §5.1: each K/V head serves a group of query
// heads), so K/V bytes are read once per K/V head, never once per query head.
//
// Per CTA: one producer warp streams 64-key stages of K and V into a shared
// memory ring with cp.async.bulk (16-byte aligned contiguous rows, completion
// on mbarriers); four consumer warps each take 16 keys of every stage:
//   A. scores: lanes split a key row into 16-byte pieces (conflict-free
//      shared loads), multiply with the pre-scaled queries held in registers,
//      and a halving shuffle reduction leaves one finished score per lane;
//   B. online softmax per row over the warp's 16 keys (running max m, sum l;
//      exp2 with scale * log2(e) folded into the queries);
//   C. weighted value sum, each lane owning R x (d / lanes-per-key) outputs.
// Warps and lanes merge their (m, l, O) at the end; with one split the CTA
// writes the normalised output, otherwise fp32 partials that the combine
// kernel merges with the log-sum-exp rule
//   O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s
// ("Causal Multi-Head Self-Attention": the Flash form keeps row maxima and
// exponential sums, which is what makes partial results mergeable).
#pragma once

#include "ptx.cuh"

namespace b200attn {

struct DecodeParams {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    float* ws_o;  // [units, nsplit, Rv, D] partial numerators (nsplit > 1)
    float* ws_m;  // [units, nsplit, Rv] running max, log2 domain
    float* ws_l;  // [units, nsplit, Rv] running sum
    int B, H, Hkv, G, Tnew, Rv;  // Rv = G * Tnew valid rows per unit
    int64_t S, S_cap, start_pos;
    int64_t kv_end;      // min(S, start_pos + Tnew): last visible key + 1
    int64_t k_lo;        // first key any row sees (0 without a local window)
    int64_t window;      // local window w: row at p sees p - w < j <= p (0: none)
    int64_t chunk;       // keys per split (multiple of the stage size)
    int nsplit;
    float scale_log2;    // scale * log2(e)
    uint64_t timeout_ns;
    uint32_t test_flags;  // kTestSkipLoads: issue no K/V copies (timeout-path tests)
    // paged cache (paged != 0): k, v are page pools [num_pages, Hkv, 2^page_shift, D];
    // page_table [B, max_pages] maps a sequence's logical page to a physical one;
    // kv_lens [B] holds each sequence's length L_b (its new tokens at L_b - Tnew ..);
    // S is then the host's bound on every L_b
    int paged;
    int page_shift;
    const int32_t* page_table;
    const int32_t* kv_lens;
    int64_t max_pages, num_pages;
};


// Positions of a unit's rows: its new tokens start at `start_pos` and the
// visible keys end at `kv_end`.  For a paged cache both come from the
// sequence's own length; a length outside [Tnew, S] is recorded in the device
// status word and clamped, so no load leaves the pool.
__device__ __forceinline__ void decode_span(const DecodeParams& p, int b, int64_t& start_pos,
                                            int64_t& kv_end) {
    if (!p.paged) {
        start_pos = p.start_pos;
        kv_end = p.kv_end;
        return;
    }
    int64_t L = p.kv_lens[b];
    if (L < p.Tnew || L > p.S) {
        atomicCAS(&g_device_status, 0u, kStatusBadIndex);
        L = max64(p.Tnew, min64(L, p.S));
    }
    start_pos = L - p.Tnew;
    kv_end = L;
}

// Issues the bulk copies of keys [k0, k0 + n) of (b, kv head) into kdst and
// vdst, completing on `bar` (which expects 2 * n * D * sizeof(T) bytes).
// Contiguous cache: one copy each, by lane 0.  Paged cache: the warp's lanes
// read the page table entries the keys span (one each, so n must span at most
// 32 pages) and lane 0 copies each page's run of rows; an entry outside the
// pool is recorded and replaced by page 0, so no load leaves the pool.
template <typename T, int D>
__device__ __forceinline__ void load_kv_rows(const DecodeParams& p, int lane, int b, int kvh,
                                             const T* kg, const T* vg, int64_t k0, int n,
                                             T* kdst, T* vdst, uint32_t bar) {
    if (!p.paged) {
        if (lane == 0) {
            const uint32_t bytes = uint32_t(n) * D * sizeof(T);
            bulk_load(smem_u32(kdst), kg + k0 * D, bytes, bar);
            bulk_load(smem_u32(vdst), vg + k0 * D, bytes, bar);
        }
        return;
    }
    const int64_t P = int64_t(1) << p.page_shift;
    const int64_t first = k0 >> p.page_shift;
    const int npg = int(((k0 + n - 1) >> p.page_shift) - first + 1);
    int64_t phys = 0;
    if (lane < npg) {
        const int64_t lp = first + lane;
        phys = lp < p.max_pages ? p.page_table[size_t(b) * p.max_pages + lp] : -1;
        if (phys < 0 || phys >= p.num_pages) {
            atomicCAS(&g_device_status, 0u, kStatusBadIndex);
            phys = 0;
        }
    }
    const T* kpool = static_cast<const T*>(p.k);
    const T* vpool = static_cast<const T*>(p.v);
    int off = 0;
    for (int pg = 0; pg < npg; ++pg) {
        const int64_t ph = __shfl_sync(0xffffffffu, phys, pg);
        const int64_t j = k0 + off;
        const int o = int(j & (P - 1));
        const int seg = int(min64(P - o, int64_t(n - off)));
        if (lane == 0) {
            const size_t row = ((size_t(ph) * p.Hkv + kvh) * size_t(P) + o) * D;
            const uint32_t bytes = uint32_t(seg) * D * sizeof(T);
            bulk_load(smem_u32(kdst + size_t(off) * D), kpool + row, bytes, bar);
            bulk_load(smem_u32(vdst + size_t(off) * D), vpool + row, bytes, bar);
        }
        off += seg;
    }
}

// Producer for a contiguous cache (lane 0 alone): stage `it` holds keys
// k_begin + it * TK .., K and V rows copied with one bulk copy each; full
// barriers bars[0..NST), empty barriers bars[NST..2 NST).
template <typename T, int D, int TK, int NST>
__device__ __forceinline__ void producer_contiguous(const DecodeParams& p, int nstages,
                                                    int64_t k_begin, int64_t k_end, const T* kg,
                                                    const T* vg, T* ks, T* vs, uint64_t* bars,
                                                    volatile int* abort_flag) {
    int issued = 0;
    const int n_loads = (p.test_flags & kTestSkipLoads) ? 0 : nstages;
    for (int it = 0; it < n_loads; ++it) {
        const int st = it % NST;
        if (!mbar_wait(smem_u32(&bars[NST + st]), ((it / NST) & 1) ^ 1, p.timeout_ns, abort_flag))
            break;
        issued = it + 1;
        const int64_t k0 = k_begin + int64_t(it) * TK;
        const int n = int(min64(TK, k_end - k0));
        const uint32_t bytes = uint32_t(n) * D * sizeof(T);
        const uint32_t full = smem_u32(&bars[st]);
        mbar_expect_tx(full, 2 * bytes);
        bulk_load(smem_u32(ks + size_t(st) * TK * D), kg + k0 * D, bytes, full);
        bulk_load(smem_u32(vs + size_t(st) * TK * D), vg + k0 * D, bytes, full);
    }
    // never leave while a copy into this CTA's shared memory is in flight
    for (int it = issued - 1; it >= 0 && it >= issued - NST; --it)
        mbar_wait(smem_u32(&bars[it % NST]), (it / NST) & 1, p.timeout_ns, nullptr);
}

template <int D, int R>
struct DecodeShape {
    static constexpr int NW = 4;                       // consumer warps
    static constexpr int TK = 64;                      // keys per stage
    static constexpr int NST = 3;                      // ring depth
    static constexpr int KW = TK / NW;                 // keys per warp per stage
    static constexpr int LPK0 = R * D / 64;
    static constexpr int LPK = LPK0 < 8 ? 8 : (LPK0 > 32 ? 32 : LPK0);  // lanes per key
    static constexpr int KPG = 32 / LPK;               // keys per warp-wide group
    static constexpr int E = D / LPK;                  // elements per lane per key
    static constexpr int CE = E >= 8 ? 8 : E;          // elements per shared load
    static constexpr int NCH = E / CE;                 // loads per lane per key
    static constexpr int GPW = KW / KPG;               // groups per warp per stage
    static constexpr int LPR = 32 / R;                 // lanes per row in the softmax step
    static constexpr int SPL = KW / LPR;               // scores per lane in that step
    static_assert(R >= 4 && R <= 32 && (R & (R - 1)) == 0, "R: power of two in [4, 32]");
    static_assert(D % (LPK * CE) == 0 && (CE == 8 || CE == 4), "head size / lane split");
    static_assert(R <= LPK, "rows must not exceed lanes per key");
    static_assert(KW % KPG == 0 && KW % LPR == 0, "stage split");
    static constexpr size_t kStageBytes(size_t esz) { return size_t(TK) * D * esz; }
    static constexpr size_t smem_bytes(size_t esz) {
        return 2 * NST * kStageBytes(esz) + size_t(NW) * KW * R * 4 + size_t(NW) * R * 4 +
               (2 * NST + 2) * 8 + 64;
    }
};

// Kernel variants: contiguous cache, paged cache, local window.
enum DecodeMode : int { kDecodePlain = 0, kDecodePaged = 1, kDecodeWindow = 2 };

template <typename T, int D, int R, int MODE>
__global__ void __launch_bounds__(160, 2)
decode_splitkv_kernel(const DecodeParams p) {
    constexpr bool PAGED = MODE == kDecodePaged;
    constexpr bool WINDOW = MODE == kDecodeWindow;
    using Sh = DecodeShape<D, R>;
    constexpr int NW = Sh::NW, TK = Sh::TK, NST = Sh::NST, KW = Sh::KW, LPK = Sh::LPK,
                  KPG = Sh::KPG, CE = Sh::CE, NCH = Sh::NCH, GPW = Sh::GPW, LPR = Sh::LPR,
                  SPL = Sh::SPL;
    extern __shared__ __align__(128) unsigned char smem[];
    T* ks = reinterpret_cast<T*>(smem);                              // [NST][TK][D]
    T* vs = ks + size_t(NST) * TK * D;                               // [NST][TK][D]
    float* sc = reinterpret_cast<float*>(vs + size_t(NST) * TK * D); // [NW][KW][R]
    float* al = sc + NW * KW * R;                                    // [NW][R]
    uint64_t* bars = reinterpret_cast<uint64_t*>(al + NW * R);       // full[NST], empty[NST]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * NST);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.y;               // b * Hkv + kvh
    const int split = blockIdx.x;
    const int b = unit / p.Hkv;
    const int kvh = unit % p.Hkv;
    int64_t start_pos = p.start_pos, kv_end = p.kv_end;
    if constexpr (PAGED) decode_span(p, b, start_pos, kv_end);
    const int64_t k_begin = (WINDOW ? p.k_lo : 0) + int64_t(split) * p.chunk;
    const int64_t k_end = min64(kv_end, k_begin + p.chunk);
    const int nstages = k_end > k_begin ? int((k_end - k_begin + TK - 1) / TK) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(smem_u32(&bars[s]), 1);
            mbar_init(smem_u32(&bars[NST + s]), NW);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // the split merge (a programmatic dependent) may be launched now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const T* kg = static_cast<const T*>(p.k) + (size_t(unit) * p.S_cap) * D;
    const T* vg = static_cast<const T*>(p.v) + (size_t(unit) * p.S_cap) * D;

    if (warp == NW) {
        // ------------------------------------------------ producer (lane 0 waits
        // and copies; for a paged cache the whole warp reads page table entries)
        if constexpr (!PAGED) {
            if (lane == 0) producer_contiguous<T, D, TK, NST>(p, nstages, k_begin, k_end, kg, vg, ks, vs,
                                                              bars, abort_flag);
            return;
        }
        int issued = 0;
        const int n_loads = (p.test_flags & kTestSkipLoads) ? 0 : nstages;
        for (int it = 0; it < n_loads; ++it) {
            const int st = it % NST;
            const uint32_t ph = (it / NST) & 1;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(smem_u32(&bars[NST + st]), ph ^ 1, p.timeout_ns, abort_flag);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            issued = it + 1;
            const int64_t k0 = k_begin + int64_t(it) * TK;
            const int n = int(min64(TK, k_end - k0));
            const uint32_t full = smem_u32(&bars[st]);
            if (lane == 0) mbar_expect_tx(full, 2 * uint32_t(n) * D * sizeof(T));
            load_kv_rows<T, D>(p, lane, b, kvh, kg, vg, k0, n, ks + size_t(st) * TK * D,
                               vs + size_t(st) * TK * D, full);
        }
        // Never leave while a copy into this CTA's shared memory is in
        // flight: wait (bounded) for the last phase issued on each stage.
        if (lane == 0)
            for (int it = issued - 1; it >= 0 && it >= issued - NST; --it)
                mbar_wait(smem_u32(&bars[it % NST]), (it / NST) & 1, p.timeout_ns, nullptr);
        return;
    }

    // ---------------------------------------------------- consumers
    const int sub = lane % LPK;        // position within the key's lane group
    const int kslot = lane / LPK;      // which key of a group this lane takes
    const int my_row = sub / (LPK / R);  // row whose finished score this lane holds

    // queries, pre-scaled into the log2 domain: qf[r][u][e]
    float qf[R][NCH][CE];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const bool valid = r < p.Rv;
        const int g = valid ? r / p.Tnew : 0;
        const int t = valid ? r % p.Tnew : 0;
        const T* qrow = static_cast<const T*>(p.q) +
                        ((size_t(b) * p.H + size_t(kvh) * p.G + g) * p.Tnew + t) * D;
#pragma unroll
        for (int u = 0; u < NCH; ++u) {
            const int e0 = (sub + LPK * u) * CE;
#pragma unroll
            for (int e = 0; e < CE; ++e)
                qf[r][u][e] = valid ? to_f32<T>(qrow[e0 + e]) * p.scale_log2 : 0.f;
        }
    }
    // causal limit of each row's position (p_i = start_pos + t)
    int64_t row_lim[R];
#pragma unroll
    for (int r = 0; r < R; ++r)
        row_lim[r] = (r < p.Rv) ? start_pos + (r % p.Tnew) : -1;
    // keys at or below row_lim[r] - wnd are outside a local window
    const int64_t wnd = WINDOW ? p.window : (int64_t(1) << 62);

    float oacc[R][NCH][CE];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int u = 0; u < NCH; ++u)
#pragma unroll
            for (int e = 0; e < CE; ++e) oacc[r][u][e] = 0.f;
    const int rb = lane / LPR;   // softmax-step row of this lane
    float m_run = -INFINITY, l_part = 0.f;
    float* scw = sc + warp * KW * R;
    float* alw = al + warp * R;

    for (int it = 0; it < nstages; ++it) {
        const int st = it % NST;
        const uint32_t ph = (it / NST) & 1;
        if (!mbar_wait(smem_u32(&bars[st]), ph, p.timeout_ns, abort_flag)) break;
        const int64_t k0 = k_begin + int64_t(it) * TK;
        const int nvalid = int(min64(TK, k_end - k0));
        const T* kst = ks + size_t(st) * TK * D;
        const T* vst = vs + size_t(st) * TK * D;

        // A. scores for this warp's KW keys
#pragma unroll
        for (int gi = 0; gi < GPW; ++gi) {
            const int kw = gi * KPG + kslot;
            const int ki = warp * KW + kw;
            const T* krow = kst + size_t(ki) * D;
            float acc[R];
#pragma unroll
            for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll
            for (int u = 0; u < NCH; ++u) {
                const int e0 = (sub + LPK * u) * CE;
                float kf[CE];
                if constexpr (CE == 8) {
                    const uint4 w = *reinterpret_cast<const uint4*>(krow + e0);
                    const float2 a = unpack2<T>(w.x), bb = unpack2<T>(w.y), c = unpack2<T>(w.z),
                                 dd = unpack2<T>(w.w);
                    kf[0] = a.x; kf[1] = a.y; kf[2] = bb.x; kf[3] = bb.y;
                    kf[4] = c.x; kf[5] = c.y; kf[6] = dd.x; kf[7] = dd.y;
                } else {
                    const uint2 w = *reinterpret_cast<const uint2*>(krow + e0);
                    const float2 a = unpack2<T>(w.x), bb = unpack2<T>(w.y);
                    kf[0] = a.x; kf[1] = a.y; kf[2] = bb.x; kf[3] = bb.y;
                }
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int e = 0; e < CE; ++e) acc[r] = fmaf(qf[r][u][e], kf[e], acc[r]);
            }
            // halving reduction over the LPK lanes of the key
            int n = R;
#pragma unroll
            for (int o = LPK / 2; o >= 1; o >>= 1) {
                if (n > 1) {
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int i = 0; i < R / 2; ++i) {
                        if (i < n / 2) {
                            const float send = upper ? acc[i] : acc[i + n / 2];
                            const float keep = upper ? acc[i + n / 2] : acc[i];
                            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                        }
                    }
                    n >>= 1;
                } else {
                    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], o);
                }
            }
            const int64_t j = k0 + ki;
            bool vis = ki < nvalid;
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (r == my_row) vis = vis && (j <= row_lim[r]) && (!WINDOW || j > row_lim[r] - wnd);
            if (sub % (LPK / R) == 0) scw[kw * R + my_row] = vis ? acc[0] : -INFINITY;
        }
        __syncwarp();

        // B. online softmax over the warp's KW keys, row rb
        {
            float s[SPL];
            float mx = -INFINITY;
#pragma unroll
            for (int e = 0; e < SPL; ++e) {
                s[e] = scw[((lane % LPR) * SPL + e) * R + rb];
                mx = fmaxf(mx, s[e]);
            }
#pragma unroll
            for (int o = LPR / 2; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m_run, mx);
            float alpha = 1.f;
            float psum = 0.f;
            if (m_new != -INFINITY) {
                alpha = ex2(m_run - m_new);
#pragma unroll
                for (int e = 0; e < SPL; ++e) {
                    s[e] = ex2(s[e] - m_new);
                    psum += s[e];
                }
            } else {
#pragma unroll
                for (int e = 0; e < SPL; ++e) s[e] = 0.f;
            }
            l_part = l_part * alpha + psum;
            m_run = m_new;
#pragma unroll
            for (int e = 0; e < SPL; ++e) scw[((lane % LPR) * SPL + e) * R + rb] = s[e];
            if (lane % LPR == 0) alw[rb] = alpha;
        }
        __syncwarp();

        // C. rescale and accumulate P V
        {
            float a[R];
            bool any = false;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                a[r] = alw[r];
                any |= (a[r] != 1.f);
            }
            if (any) {
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int u = 0; u < NCH; ++u)
#pragma unroll
                        for (int e = 0; e < CE; ++e) oacc[r][u][e] *= a[r];
            }
#pragma unroll
            for (int gi = 0; gi < GPW; ++gi) {
                const int kw = gi * KPG + kslot;
                const int ki = warp * KW + kw;
                if (ki < nvalid) {
                    float pr[R];
#pragma unroll
                    for (int r = 0; r < R; ++r) pr[r] = scw[kw * R + r];
                    const T* vrow = vst + size_t(ki) * D;
#pragma unroll
                    for (int u = 0; u < NCH; ++u) {
                        const int e0 = (sub + LPK * u) * CE;
                        float vf[CE];
                        if constexpr (CE == 8) {
                            const uint4 w = *reinterpret_cast<const uint4*>(vrow + e0);
                            const float2 x0 = unpack2<T>(w.x), x1 = unpack2<T>(w.y),
                                         x2 = unpack2<T>(w.z), x3 = unpack2<T>(w.w);
                            vf[0] = x0.x; vf[1] = x0.y; vf[2] = x1.x; vf[3] = x1.y;
                            vf[4] = x2.x; vf[5] = x2.y; vf[6] = x3.x; vf[7] = x3.y;
                        } else {
                            const uint2 w = *reinterpret_cast<const uint2*>(vrow + e0);
                            const float2 x0 = unpack2<T>(w.x), x1 = unpack2<T>(w.y);
                            vf[0] = x0.x; vf[1] = x0.y; vf[2] = x1.x; vf[3] = x1.y;
                        }
#pragma unroll
                        for (int r = 0; r < R; ++r)
#pragma unroll
                            for (int e = 0; e < CE; ++e)
                                oacc[r][u][e] = fmaf(pr[r], vf[e], oacc[r][u][e]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars[NST + st]));
    }

    // ---------------------------------------------------- merge
    // lanes holding different keys of a group hold partial sums of the same outputs
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1)
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int u = 0; u < NCH; ++u)
#pragma unroll
                for (int e = 0; e < CE; ++e)
                    oacc[r][u][e] += __shfl_xor_sync(0xffffffffu, oacc[r][u][e], o);
#pragma unroll
    for (int o = LPR / 2; o >= 1; o >>= 1) l_part += __shfl_xor_sync(0xffffffffu, l_part, o);

    // all consumer warps are past their last full-barrier wait: the ring is idle
    asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
    float* mo = reinterpret_cast<float*>(smem);  // [NW][R]
    float* lo = mo + NW * R;                     // [NW][R]
    float* oo = lo + NW * R;                     // [NW][R][D]
    if (lane % LPR == 0) {
        mo[warp * R + rb] = m_run;
        lo[warp * R + rb] = l_part;
    }
    if (kslot == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int u = 0; u < NCH; ++u)
#pragma unroll
                for (int e = 0; e < CE; ++e)
                    oo[(warp * R + r) * D + (sub + LPK * u) * CE + e] = oacc[r][u][e];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");

    const bool aborted = *abort_flag != 0;
    for (int idx = threadIdx.x; idx < p.Rv * D; idx += NW * 32) {
        const int r = idx / D, e = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, mo[w * R + r]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = ex2(mo[w * R + r] - M);
                L += f * lo[w * R + r];
                acc += f * oo[(w * R + r) * D + e];
            }
        }
        if (aborted) continue;
        if (p.nsplit == 1) {
            const int g = r / p.Tnew, t = r % p.Tnew;
            const size_t orow = (size_t(b) * p.H + size_t(kvh) * p.G + g) * p.Tnew + t;
            static_cast<T*>(p.o)[orow * D + e] = from_f32<T>(L > 0.f ? acc / L : 0.f);
            if (e == 0 && p.lse)
                p.lse[orow] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
        } else {
            const size_t pi = (size_t(unit) * p.nsplit + split) * p.Rv + r;
            p.ws_o[pi * D + e] = acc;
            if (e == 0) {
                p.ws_m[pi] = M;
                p.ws_l[pi] = L;
            }
        }
    }
}

// Merge split partials: one warp per output row (unit, r).
template <typename T, int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(const DecodeParams p) {
    // launched as a programmatic dependent of the decode kernel: its launch
    // overlaps the decode's tail, and this wait holds it until the decode
    // grid has finished and its partials are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = int64_t(blockIdx.x) * 4 + warp;  // over units * Rv
    const int64_t nrows = int64_t(p.B) * p.Hkv * p.Rv;
    if (row >= nrows) return;
    const int unit = int(row / p.Rv), r = int(row % p.Rv);
    float M = -INFINITY;
    for (int s = 0; s < p.nsplit; ++s)
        M = fmaxf(M, p.ws_m[(size_t(unit) * p.nsplit + s) * p.Rv + r]);
    constexpr int C = (D + 31) / 32;
    float acc[C];
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = 0.f;
    float L = 0.f;
    for (int s = 0; s < p.nsplit; ++s) {
        const size_t pi = (size_t(unit) * p.nsplit + s) * p.Rv + r;
        const float ms = p.ws_m[pi];
        if (ms == -INFINITY) continue;
        const float f = ex2(ms - M);
        L += f * p.ws_l[pi];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            const int e = lane + 32 * c;
            if (e < D) acc[c] = fmaf(f, p.ws_o[pi * D + e], acc[c]);
        }
    }
    const int b = unit / p.Hkv, kvh = unit % p.Hkv;
    const int g = r / p.Tnew, t = r % p.Tnew;
    const size_t orow = (size_t(b) * p.H + size_t(kvh) * p.G + g) * p.Tnew + t;
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const int e = lane + 32 * c;
        if (e < D) static_cast<T*>(p.o)[orow * D + e] = from_f32<T>(acc[c] * inv);
    }
    if (lane == 0 && p.lse)
        p.lse[orow] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace b200attn
