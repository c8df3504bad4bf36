// CUDA-core backward pass: the float32 path, and 16-bit head sizes the
// tensor-core backward kernels do not take (any d up to 256).
//
// Same mathematics as the tensor-core kernels ("Causal Multi-Head
// Self-Attention", Two exact full-sequence algorithms: probabilities rebuilt
// from Q, K and the saved row statistic, then the exact softmax
// vector-Jacobian product), with every step in float32 and the accurate
// exp2f:
//   simt_bwd_dkdv   one warp per key row (b, K/V head, j): walks the query
//                   rows of every query head of the group that see the key,
//                   accumulating dV_j = sum P_ij dO_i and
//                   dK_j = scale * sum dS_ij Q_i in registers;
//   simt_bwd_dq     one warp per query row (b, h, i): walks the keys it sees,
//                   dQ_i = scale * sum_j dS_ij K_j.
// Lanes own the head dimension (column t on lane t % 32); dot products end
// in a butterfly reduction.  The row terms D_i and -lse_i * log2(e) come from
// bwd_preprocess_kernel.
#pragma once

#include "prefill_backward.cuh"

namespace b200attn {

constexpr int kSimtBwdWarps = 4;
constexpr int kSimtBwdCols = 8;   // columns per lane: d <= 256

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

template <typename T>
__device__ __forceinline__ void load_row(const T* src, int d, int lane, float (&r)[kSimtBwdCols]) {
#pragma unroll
    for (int c = 0; c < kSimtBwdCols; ++c) {
        const int t = lane + 32 * c;
        r[c] = t < d ? to_f32<T>(src[t]) : 0.f;
    }
}

template <typename T>
__device__ __forceinline__ void store_row(T* dst, int d, int lane, const float (&r)[kSimtBwdCols], float mul) {
#pragma unroll
    for (int c = 0; c < kSimtBwdCols; ++c) {
        const int t = lane + 32 * c;
        if (t < d) dst[t] = from_f32<T>(r[c] * mul);
    }
}

__device__ __forceinline__ float dot_row(const float (&a)[kSimtBwdCols], const float (&b)[kSimtBwdCols]) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kSimtBwdCols; ++c) s = fmaf(a[c], b[c], s);
    return warp_sum(s);
}

// Q, K and V (the tensor-core kernels read them through tensor maps instead).
struct SimtBwdPtrs {
    const void* q;
    const void* k;
    const void* v;
};

template <typename T>
__global__ void __launch_bounds__(kSimtBwdWarps * 32)
simt_bwd_dkdv_kernel(const BwdParams p, const SimtBwdPtrs in) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = int64_t(blockIdx.x) * kSimtBwdWarps + warp;   // (b, kvh, j)
    if (row >= int64_t(p.B) * p.Hkv * p.T) return;
    const int j = int(row % p.T);
    const int64_t bk = row / p.T;
    const int b = int(bk / p.Hkv), kvh = int(bk % p.Hkv);
    float kr[kSimtBwdCols], vr[kSimtBwdCols], dk[kSimtBwdCols], dv[kSimtBwdCols];
    load_row<T>(static_cast<const T*>(in.k) + size_t(row) * p.d, p.d, lane, kr);
    load_row<T>(static_cast<const T*>(in.v) + size_t(row) * p.d, p.d, lane, vr);
#pragma unroll
    for (int c = 0; c < kSimtBwdCols; ++c) dk[c] = dv[c] = 0.f;
    const float c2 = p.scale_log2;
    for (int g = 0; g < p.G; ++g) {
        const int64_t bh = int64_t(b) * p.H + int64_t(kvh) * p.G + g;
        const T* qb = static_cast<const T*>(in.q) + size_t(bh) * p.T * p.d;
        const T* gb = static_cast<const T*>(p.dout) + size_t(bh) * p.T * p.d;
        const float* nl = p.nl + size_t(bh) * p.Tpad;
        const float* dd = p.dd + size_t(bh) * p.Tpad;
        const int i_end = p.window > 0 ? min(p.T, j + p.window) : p.T;
        for (int i = p.causal ? j : 0; i < i_end; ++i) {
            float qr[kSimtBwdCols], gr[kSimtBwdCols];
            load_row<T>(qb + size_t(i) * p.d, p.d, lane, qr);
            load_row<T>(gb + size_t(i) * p.d, p.d, lane, gr);
            const float P = exp2f(fmaf(dot_row(qr, kr), c2, nl[i]));
            const float dS = P * (dot_row(gr, vr) - dd[i]);
#pragma unroll
            for (int c = 0; c < kSimtBwdCols; ++c) {
                dv[c] = fmaf(P, gr[c], dv[c]);
                dk[c] = fmaf(dS, qr[c], dk[c]);
            }
        }
    }
    store_row<T>(static_cast<T*>(p.dv) + size_t(row) * p.d, p.d, lane, dv, 1.f);
    store_row<T>(static_cast<T*>(p.dk) + size_t(row) * p.d, p.d, lane, dk, p.scale);
}

template <typename T>
__global__ void __launch_bounds__(kSimtBwdWarps * 32)
simt_bwd_dq_kernel(const BwdParams p, const SimtBwdPtrs in) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = int64_t(blockIdx.x) * kSimtBwdWarps + warp;   // (b, h, i)
    if (row >= int64_t(p.B) * p.H * p.T) return;
    const int i = int(row % p.T);
    const int64_t bh = row / p.T;
    const int b = int(bh / p.H), h = int(bh % p.H);
    const int64_t bk = int64_t(b) * p.Hkv + h / p.G;
    float qr[kSimtBwdCols], gr[kSimtBwdCols], dq[kSimtBwdCols];
    load_row<T>(static_cast<const T*>(in.q) + size_t(row) * p.d, p.d, lane, qr);
    load_row<T>(static_cast<const T*>(p.dout) + size_t(row) * p.d, p.d, lane, gr);
#pragma unroll
    for (int c = 0; c < kSimtBwdCols; ++c) dq[c] = 0.f;
    const float nl = p.nl[size_t(bh) * p.Tpad + i];
    const float dd = p.dd[size_t(bh) * p.Tpad + i];
    const float c2 = p.scale_log2;
    const T* kb = static_cast<const T*>(in.k) + size_t(bk) * p.T * p.d;
    const T* vb = static_cast<const T*>(in.v) + size_t(bk) * p.T * p.d;
    const int j_end = p.causal ? i + 1 : p.T;
    for (int j = p.window > 0 ? max(0, i - p.window + 1) : 0; j < j_end; ++j) {
        float kr[kSimtBwdCols], vr[kSimtBwdCols];
        load_row<T>(kb + size_t(j) * p.d, p.d, lane, kr);
        load_row<T>(vb + size_t(j) * p.d, p.d, lane, vr);
        const float P = exp2f(fmaf(dot_row(qr, kr), c2, nl));
        const float dS = P * (dot_row(gr, vr) - dd);
#pragma unroll
        for (int c = 0; c < kSimtBwdCols; ++c) dq[c] = fmaf(dS, kr[c], dq[c]);
    }
    store_row<T>(static_cast<T*>(p.dq) + size_t(row) * p.d, p.d, lane, dq, p.scale);
}

// D and -lse*log2(e) for every row of [B*H, Tpad] (any d, any element type).
template <typename T>
__global__ void __launch_bounds__(kSimtBwdWarps * 32) simt_bwd_preprocess_kernel(const BwdParams p) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t r = int64_t(blockIdx.x) * kSimtBwdWarps + warp;
    if (r >= int64_t(p.B) * p.H * p.Tpad) return;
    const int64_t bh = r / p.Tpad;
    const int i = int(r - bh * p.Tpad);
    float acc = 0.f;
    if (i < p.T) {
        const size_t off = (size_t(bh) * p.T + i) * p.d;
        const T* o = static_cast<const T*>(p.o) + off;
        const T* g = static_cast<const T*>(p.dout) + off;
        for (int t = lane; t < p.d; t += 32) acc = fmaf(to_f32<T>(o[t]), to_f32<T>(g[t]), acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
        p.dd[r] = i < p.T ? acc : 0.f;
        p.nl[r] = i < p.T ? -p.lse[size_t(bh) * p.T + i] * 1.4426950408889634f : -INFINITY;
    }
}

}  // namespace b200attn
