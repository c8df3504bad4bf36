// KV-cache append with rotary position embedding on K: the step directly
// before cached attention ("Hesper.Layers.Attention", the fused RoPE-K and
// cache-write kernels: rotate the new K with the NeoX pairing — dimension i
// turns with i + d/2 — and write K and V into the cache rows of their
// positions; "Grouped-Query Attention" §5.1: apply_rope at offset start_pos,
// then the cache append).  HBM-bound: every byte read once, written once.
//
// One CTA per (b, group of up to kAppendMaxTok consecutive new tokens).  The
// work is cut into units: a unit is KB bytes (16 or 8) of the first half of
// one K or V row together with the KB bytes of the second half that K pairs
// them with.  Each thread issues the loads of kAppendUnits units before it
// touches any of them; on the first round the CTA then builds the cos / sin
// tables of its tokens' positions p = start_pos + t (angle p * inv_freq[i]
// formed and reduced mod 2*pi in fp64, then fp32 sincos), so
// the tables' latency hides under the loads.  The rotation runs on packed
// float2 FMAs; unit indices are split with multiply-shift division.
#pragma once

#include "ptx.cuh"

namespace b200attn {

constexpr int kAppendMaxD = 256;
constexpr int kAppendMaxTok = 8;     // tokens per CTA
constexpr int kAppendUnits = 2;      // units in flight per thread (2: 5.70 TB/s, 4: 5.57, 8: 5.24 on the GQA rows)

// Division by a fixed divisor n >= 1 for numerators below 2^31, by multiply
// and shift (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): q = (umulhi(x, mul) + x) >> shift, with
// shift = ceil(log2 n) and mul = floor(2^32 (2^shift - n) / n) + 1.
struct FastDiv {
    uint32_t n, mul, shift;
    __host__ __device__ FastDiv() : n(1), mul(0), shift(0) {}
    __host__ explicit FastDiv(uint32_t divisor) : n(divisor) {
        shift = 0;
        while ((uint64_t(1) << shift) < divisor) ++shift;
        mul = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << shift) - divisor)) / divisor + 1);
    }
    __device__ __forceinline__ uint32_t div(uint32_t x) const {
        return (__umulhi(x, mul) + x) >> shift;
    }
};

struct AppendParams {
    const void* k_new;   // [B, Hkv, Tnew, d]
    const void* v_new;   // [B, Hkv, Tnew, d]
    void* k_cache;       // [B, Hkv, S_cap, d]
    void* v_cache;       // [B, Hkv, S_cap, d]
    int B, Hkv, Tnew, d;
    int64_t S_cap, start_pos;
    int rotate;          // 0: plain append
    int tok_per_cta;     // tokens per CTA, <= kAppendMaxTok
    int half_units;      // d/2 * esz / KB: units per row
    FastDiv div_tok;     // by 2 * Hkv * half_units: units per token
    FastDiv div_row;     // by half_units
    double inv_freq[kAppendMaxD / 2];   // base^(-2i/d), i < d/2
};

template <int KB> struct KVec;
template <> struct KVec<16> { using type = uint4; };
template <> struct KVec<8> { using type = uint2; };

// Rotates the pairs held by a first-half vector `lo` and its second-half
// partner `hi`: x0' = x0 cos - x1 sin, x1' = x1 cos + x0 sin, element j of the
// vectors turning by the angle of pair i0 + j.  `cs`, `sn`, `ns` are the
// token's cos, sin and -sin rows.
template <typename T, int KB>
__device__ __forceinline__ void rotate_vec(typename KVec<KB>::type& lo, typename KVec<KB>::type& hi,
                                           int i0, const float* cs, const float* sn,
                                           const float* ns) {
    uint32_t* a = reinterpret_cast<uint32_t*>(&lo);
    uint32_t* b = reinterpret_cast<uint32_t*>(&hi);
    constexpr int W = KB / 4;   // 32-bit words per vector
    if constexpr (std::is_same<T, float>::value) {
#pragma unroll
        for (int w = 0; w < W; w += 2) {
            const float2 x0 = make_float2(__uint_as_float(a[w]), __uint_as_float(a[w + 1]));
            const float2 x1 = make_float2(__uint_as_float(b[w]), __uint_as_float(b[w + 1]));
            const float2 c = *reinterpret_cast<const float2*>(cs + i0 + w);
            const float2 s = *reinterpret_cast<const float2*>(sn + i0 + w);
            const float2 n = *reinterpret_cast<const float2*>(ns + i0 + w);
            const float2 y0 = __ffma2_rn(x1, n, __fmul2_rn(x0, c));
            const float2 y1 = __ffma2_rn(x0, s, __fmul2_rn(x1, c));
            a[w] = __float_as_uint(y0.x); a[w + 1] = __float_as_uint(y0.y);
            b[w] = __float_as_uint(y1.x); b[w + 1] = __float_as_uint(y1.y);
        }
    } else {
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const float2 x0 = unpack2<T>(a[w]), x1 = unpack2<T>(b[w]);
            const float2 c = *reinterpret_cast<const float2*>(cs + i0 + 2 * w);
            const float2 s = *reinterpret_cast<const float2*>(sn + i0 + 2 * w);
            const float2 n = *reinterpret_cast<const float2*>(ns + i0 + 2 * w);
            const float2 y0 = __ffma2_rn(x1, n, __fmul2_rn(x0, c));
            const float2 y1 = __ffma2_rn(x0, s, __fmul2_rn(x1, c));
            a[w] = pack2<T>(y0.x, y0.y);
            b[w] = pack2<T>(y1.x, y1.y);
        }
    }
}

template <int KB>
struct AppendUnit {
    typename KVec<KB>::type lo, hi;   // matching vectors of the two halves of a row
};

template <typename T, int KB>
__global__ void __launch_bounds__(256)
kv_append_rope_kernel(const __grid_constant__ AppendParams p) {
    using KV = typename KVec<KB>::type;
    constexpr int E = KB / int(sizeof(T));   // elements per vector
    constexpr int TS = kAppendMaxD / 2;      // table row stride
    __shared__ __align__(16) float cs[kAppendMaxTok * TS], sn[kAppendMaxTok * TS],
        ns[kAppendMaxTok * TS];
    const int groups = (p.Tnew + p.tok_per_cta - 1) / p.tok_per_cta;
    const int b = blockIdx.x / groups;
    const int t0 = (blockIdx.x % groups) * p.tok_per_cta;
    const int ntok = min(p.tok_per_cta, p.Tnew - t0);
    const int k_units = p.Hkv * p.half_units;       // per token; as many V units follow
    const int total = ntok * 2 * k_units;
    const int h = p.d / 2;
    const size_t in_base = size_t(b) * p.Hkv * p.Tnew + t0;
    const size_t out_base = size_t(b) * p.Hkv * p.S_cap + p.start_pos + t0;
    for (int base = 0; base < total; base += kAppendUnits * blockDim.x) {
        AppendUnit<KB> x[kAppendUnits];
        KV* dst[kAppendUnits];
        int tab[kAppendUnits];   // table offset of a K unit's first pair; -1 for V
#pragma unroll
        for (int j = 0; j < kAppendUnits; ++j) {
            const int u = base + j * blockDim.x + threadIdx.x;
            dst[j] = nullptr;
            tab[j] = -1;
            if (u < total) {
                const int tok = int(p.div_tok.div(uint32_t(u)));
                int r = u - tok * 2 * k_units;
                const bool is_v = r >= k_units;
                if (is_v) r -= k_units;
                const int kv = int(p.div_row.div(uint32_t(r)));
                const int c = r - kv * p.half_units;
                const size_t in_row = (in_base + size_t(kv) * p.Tnew + tok) * p.d;
                const size_t out_row = (out_base + size_t(kv) * p.S_cap + tok) * p.d;
                const KV* src = reinterpret_cast<const KV*>(
                    static_cast<const T*>(is_v ? p.v_new : p.k_new) + in_row) + c;
                x[j].lo = src[0];
                x[j].hi = src[p.half_units];
                dst[j] = reinterpret_cast<KV*>(static_cast<T*>(is_v ? p.v_cache : p.k_cache) +
                                               out_row) + c;
                if (!is_v && p.rotate) tab[j] = tok * TS + c * E;
            }
        }
        if (base == 0 && p.rotate) {
            constexpr double kTwoPiHi = 6.283185307179586;
            constexpr double kTwoPiLo = 2.4492935982947064e-16;
            for (int e = threadIdx.x; e < ntok * h; e += blockDim.x) {
                const int tok = e / h, i = e - tok * h;
                const double ang = double(p.start_pos + t0 + tok) * p.inv_freq[i];
                const double k = rint(ang * (1.0 / kTwoPiHi));
                const float r = float(fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, ang)));   // |r| <= pi
                float sv, cv;
                sincosf(r, &sv, &cv);
                cs[tok * TS + i] = cv;
                sn[tok * TS + i] = sv;
                ns[tok * TS + i] = -sv;
            }
            __syncthreads();
        }
#pragma unroll
        for (int j = 0; j < kAppendUnits; ++j) {
            if (dst[j] == nullptr) continue;
            if (tab[j] >= 0) rotate_vec<T, KB>(x[j].lo, x[j].hi, tab[j], cs, sn, ns);
            dst[j][0] = x[j].lo;
            dst[j][p.half_units] = x[j].hi;
        }
    }
}

}  // namespace b200attn
