// CUDA-core attention kernel: the float32 path, and any head size up to 256
// for 16-bit inputs whose shape the tensor-core kernels do not take.
//
// One warp owns one query row (b, h, i).  It walks the visible keys in blocks
// of 32 (one key per lane), keeps a running row maximum m and normaliser l
// ("Causal Multi-Head Self-Attention", Two exact full-sequence algorithms:
// the Flash form saves only row maxima and exponential sums and rescales as
// each key tile arrives), and accumulates the weighted values with each lane
// owning d/32 output columns.  Exponentials use expf in the natural-log
// domain so the float32 path keeps float32 accuracy.
#pragma once

#include "ptx.cuh"

namespace b200attn {

struct SimtParams {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    int64_t B, H, Hkv, Tq, S, S_cap, d, start_pos;
    float scale;
    int causal;
    int64_t window;  // local window w: the row at p sees p - w < j <= p (0: none)
};

constexpr int kSimtWarps = 4;
constexpr int kSimtMaxD = 256;

template <typename T>
__global__ void __launch_bounds__(kSimtWarps * 32)
simt_attention_kernel(const SimtParams p) {
    __shared__ float q_sh[kSimtWarps][kSimtMaxD];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kSimtWarps + warp;
    const int64_t nrows = p.B * p.H * p.Tq;
    if (row >= nrows) return;

    const int64_t i = row % p.Tq;
    const int64_t h = (row / p.Tq) % p.H;
    const int64_t b = row / (p.Tq * p.H);
    const int64_t kvh = h / (p.H / p.Hkv);
    const int d = static_cast<int>(p.d);
    const T* qrow = static_cast<const T*>(p.q) + row * p.d;
    const T* kbase = static_cast<const T*>(p.k) + (b * p.Hkv + kvh) * p.S_cap * p.d;
    const T* vbase = static_cast<const T*>(p.v) + (b * p.Hkv + kvh) * p.S_cap * p.d;

    for (int t = lane; t < d; t += 32) q_sh[warp][t] = to_f32<T>(qrow[t]);
    __syncwarp();

    const int64_t pos = p.start_pos + i;
    const int64_t kv_end = p.causal ? min(p.S, pos + 1) : p.S;
    const int64_t kv_lo = p.window > 0 ? max(int64_t(0), pos - p.window + 1) : int64_t(0);

    constexpr int kCols = kSimtMaxD / 32;
    float acc[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) acc[c] = 0.f;
    float m = -INFINITY, l = 0.f;

    for (int64_t j0 = kv_lo; j0 < kv_end; j0 += 32) {
        const int64_t j = j0 + lane;
        float s = -INFINITY;
        if (j < kv_end) {
            const T* krow = kbase + j * p.d;
            float dot = 0.f;
            for (int t = 0; t < d; ++t) dot = fmaf(q_sh[warp][t], to_f32<T>(krow[t]), dot);
            s = dot * p.scale;
        }
        float mx = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m, mx);  // finite: key j0 is always visible
        const float alpha = expf(m - m_new);
        const float pj = (j < kv_end) ? expf(s - m_new) : 0.f;
        float psum = pj;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l = l * alpha + psum;
        m = m_new;
#pragma unroll
        for (int c = 0; c < kCols; ++c) acc[c] *= alpha;
        const int nk = static_cast<int>(min64(32, kv_end - j0));
        for (int kk = 0; kk < nk; ++kk) {
            const float w = __shfl_sync(0xffffffffu, pj, kk);
            const T* vrow = vbase + (j0 + kk) * p.d;
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const int t = lane + 32 * c;
                if (t < d) acc[c] = fmaf(w, to_f32<T>(vrow[t]), acc[c]);
            }
        }
    }

    T* orow = static_cast<T*>(p.o) + row * p.d;
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
        const int t = lane + 32 * c;
        if (t < d) orow[t] = from_f32<T>(acc[c] * inv);
    }
    if (p.lse && lane == 0) p.lse[row] = (l > 0.f) ? m + logf(l) : -INFINITY;
}

}  // namespace b200attn
