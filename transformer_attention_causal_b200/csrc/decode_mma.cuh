// Split-KV cached decode on warp-level tensor-core MMAs (d a multiple of 16
// in [64, 128], up to 16 rows per K/V head; contiguous or paged cache).
//
// Same split, online softmax and merge as decode_splitkv_kernel ("Multi-query
// attention, annotated" §2.4.1: the call streams the visible history once,
// so it is bound by HBM), with the per-key arithmetic moved off the FMA pipes:
// the CUDA-core kernels spend ~64 warp instructions per key on widening,
// packed FMAs and shuffle reductions, which leaves them ~20 % short of the
// bytes HBM can deliver.  Here a warp takes 16 keys of every 128-key stage:
//   S^T (16 keys x 8 rows) = K Q^T   mma.m16n8k16: K from shared memory
//                                     (ldmatrix), Q held in registers as the
//                                     B fragments (the rows padded to 8);
//   online softmax per row            each row's 16 scores sit on 8 lanes:
//                                     three butterfly steps give the block
//                                     maximum; the running maximum is raised
//                                     lazily (by more than 2^8 only);
//   P^T                               the score fragment rounded to 16 bits
//                                     and transposed in registers (movmatrix)
//                                     is exactly the B fragment of
//   O^T (d x 8 rows) += V^T P^T       mma.m16n8k16 with V^T from ldmatrix.trans.
// About four instructions per key.  K and V stages arrive by TMA with the
// 128-byte swizzle (conflict-free ldmatrix rows); rows past the end of the
// history are zero-filled by TMA and masked by position.  A head size that is
// not a multiple of 64 fills its last 64-column chunk partly (TMA zero-fills
// the rest) and runs d / 16 k-steps and m-tiles.
// Paged variant: each 128-key stage is one TMA copy per page it spans (boxes
// of min(P, 128) rows over the pools); rows past the sequence's end and
// out-of-range page ids (reported) are read at an out-of-range coordinate and
// come back zero-filled, and the rows of the sequence's last page past its
// length, which a whole-page copy brings in, are zeroed in shared memory by
// the warp that owns them before any MMA reads them.
#pragma once

#include "decode_splitkv.cuh"

namespace b200attn {

constexpr int kDecMmaWarps = 8;                     // consumer warps (16 keys each per stage)
constexpr int kDecMmaTK = 16 * kDecMmaWarps;        // keys per stage
constexpr int kDecMmaThreads = 32 * (kDecMmaWarps + 1);

template <int DCH> struct DecMmaShape {
    static constexpr int NST = DCH == 2 ? 3 : 6;    // ring depth: 192 KB either way
    static constexpr uint32_t TB = DCH * 16384u;    // one 128-key tile of K or V
    static constexpr size_t smem_bytes() { return 1024 + size_t(NST) * 2 * TB + 256; }
};

// Shared address of (key row `key`, column d0) in a 128-row tile of DCH
// 64-column chunks written by TMA with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_addr(uint32_t tile, int key, int d0) {
    const int u = (d0 & 63) >> 3;
    return tile + uint32_t(d0 >> 6) * 16384u + uint32_t(key) * 128u + (uint32_t(u ^ (key & 7)) << 4);
}

template <typename T, int D, int NT, bool WINDOW, bool PAGED>
__global__ void __launch_bounds__(kDecMmaThreads, 1)
decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
    static_assert(D % 16 == 0 && D >= 64 && D <= 128, "head size");
    constexpr int DCH = (D + 63) / 64;          // 64-column chunks of a K/V row
    constexpr int NK = D / 16;                  // k-steps of S^T, m-tiles of O^T
    constexpr int NW = kDecMmaWarps, TK = kDecMmaTK;
    constexpr int NST = DecMmaShape<DCH>::NST;
    constexpr uint32_t TB = DecMmaShape<DCH>::TB;
    constexpr int RM = 8 * NT;                  // padded rows
    extern __shared__ unsigned char smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char* base_ptr = smem_raw + (base - smem_u32(smem_raw));
    uint64_t* bars = reinterpret_cast<uint64_t*>(base_ptr + size_t(NST) * 2 * TB);   // full[NST], empty[NST]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * NST);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.y;
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
    // the split merge (a programmatic dependent) may be launched now; it
    // waits for this grid to finish before it reads anything
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == NW) {
        // ============================================ TMA producer (lane 0)
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued = 0;
            const int n_loads = (p.test_flags & kTestSkipLoads) ? 0 : nstages;
            for (int it = 0; it < n_loads; ++it) {
                const int st = it % NST;
                if (!mbar_wait(smem_u32(&bars[NST + st]), ((it / NST) & 1) ^ 1, p.timeout_ns, abort_flag))
                    break;
                const uint32_t full = smem_u32(&bars[st]);
                mbar_expect_tx(full, 2 * TB);
                const int32_t k0 = int32_t(k_begin + int64_t(it) * TK);
                const uint32_t kt = base + uint32_t(st) * 2 * TB;
                if constexpr (PAGED) {
                    const int rows = min(1 << p.page_shift, TK);
                    for (int sub = 0; sub < TK / rows; ++sub) {
                        const int64_t tok = int64_t(k0) + int64_t(sub) * rows;
                        int64_t z = p.num_pages * p.Hkv;   // past the pools: zero fill
                        int y = 0;
                        if (tok < kv_end) {
                            const int32_t phys = p.page_table[int64_t(b) * p.max_pages + (tok >> p.page_shift)];
                            if (phys < 0 || phys >= p.num_pages) {
                                atomicCAS(&g_device_status, 0u, kStatusBadIndex);
                            } else {
                                z = int64_t(phys) * p.Hkv + kvh;
                                y = int(tok & ((int64_t(1) << p.page_shift) - 1));
                            }
                        }
                        const uint32_t off = uint32_t(sub * rows) * 128u;
                        for (int c = 0; c < DCH; ++c) {
                            tma_load_3d(kt + c * 16384u + off, &tmK, full, c * 64, y, int32_t(z));
                            tma_load_3d(kt + TB + c * 16384u + off, &tmV, full, c * 64, y, int32_t(z));
                        }
                    }
                } else {
                    for (int c = 0; c < DCH; ++c) {
                        tma_load_3d(kt + c * 16384u, &tmK, full, c * 64, k0, unit);
                        tma_load_3d(kt + TB + c * 16384u, &tmV, full, c * 64, k0, unit);
                    }
                }
                issued = it + 1;
            }
            for (int it = issued - 1; it >= 0 && it >= issued - NST; --it)
                mbar_wait(smem_u32(&bars[it % NST]), (it / NST) & 1, p.timeout_ns, nullptr);
        }
        return;
    }

    // ================================================ consumers
    const int kb = warp * 16;                  // this warp's 16 keys within a stage
    const int rsub = (lane & 3) * 2;           // the two rows (per n-tile) this lane holds
    // Q^T as B fragments: row n = lane / 4 (+ 8 nt), d pairs (lane % 4) * 2 (+ 8)
    uint32_t qf[NT][NK][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int r = nt * 8 + lane / 4;
        const bool valid = r < p.Rv;
        const int g = valid ? r / p.Tnew : 0, t = valid ? r % p.Tnew : 0;
        const T* qrow = static_cast<const T*>(p.q) + ((size_t(b) * p.H + size_t(kvh) * p.G + g) * p.Tnew + t) * D;
#pragma unroll
        for (int kk = 0; kk < NK; ++kk) {
            const int d0 = kk * 16 + rsub;
            qf[nt][kk][0] = valid ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
            qf[nt][kk][1] = valid ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 8) : 0u;
        }
    }
    const bool single = p.Tnew == 1;
    int64_t lim[NT][2];
    bool rvalid[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int r = nt * 8 + rsub + rr;
            rvalid[nt][rr] = r < p.Rv;
            lim[nt][rr] = start_pos + (r % p.Tnew);
        }
    float m_run[NT][2], l_part[NT][2];
    float o[NT][NK][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_part[nt][0] = l_part[nt][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < NK; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    }
    const float c2 = p.scale_log2;
    // ldmatrix lane roles: matrix l / 8, its row l % 8
    const int mi = lane >> 3, mrow = lane & 7;

    for (int it = 0; it < nstages; ++it) {
        const int st = it % NST;
        if (!mbar_wait(smem_u32(&bars[st]), (it / NST) & 1, p.timeout_ns, abort_flag)) break;
        const int64_t k0 = k_begin + int64_t(it) * TK;
        const uint32_t ks = base + uint32_t(st) * 2 * TB, vs = ks + TB;
        if constexpr (PAGED) {
            // V rows of this warp past the sequence's end: a whole-page copy may
            // have brought in whatever the page holds there; their P is 0, so
            // make them 0 too (0 * NaN would not be)
            const int64_t first_bad = k_end - (k0 + kb);
            if (first_bad < 16) {
                for (int idx = lane; idx < 16 * DCH * 8; idx += 32) {
                    const int key = idx / (DCH * 8);
                    if (key < first_bad) continue;
                    const int u = idx % (DCH * 8);
                    const uint32_t a = vs + uint32_t(u >> 3) * 16384u + uint32_t(kb + key) * 128u + uint32_t(u & 7) * 16u;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                }
                // ordered before the TMA refill of this stage (async proxy)
                fence_proxy_async_smem();
                __syncwarp();
            }
        }

        // ---- S^T = K Q^T (fp32, 16 keys x RM rows)
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < NK; ++kk) {
            uint32_t a[4];
            ldsm_x4(sw128_addr(ks, kb + mrow + (mi & 1) * 8, kk * 16 + (mi >> 1) * 8), a);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_16816<T>(s[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
        }

        // ---- scale and mask: s[nt][e] is key kb + lane/4 (+ 8 for e >= 2), row rsub + (e & 1)
        const int64_t j0 = k0 + kb + lane / 4;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t j = j0 + (e >> 1) * 8;
                const int rr = e & 1;
                bool vis = j < k_end && rvalid[nt][rr];
                if (!single) vis = vis && j <= lim[nt][rr] && (!WINDOW || j > lim[nt][rr] - p.window);
                s[nt][e] = vis ? s[nt][e] * c2 : -INFINITY;
            }

        // ---- online softmax: block maximum over the 8 lanes that share a row pair
        bool need_any = false;
        float bm[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                float m = fmaxf(s[nt][rr], s[nt][rr + 2]);
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
                bm[nt][rr] = m;
                need_any |= m - m_run[nt][rr] > 8.f;   // -inf - -inf = NaN: false
            }
        if (__any_sync(0xffffffffu, need_any)) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    if (!(bm[nt][rr] - m_run[nt][rr] > 8.f)) continue;
                    const float alpha = ex2(m_run[nt][rr] - bm[nt][rr]);   // 0 for the first keys
                    m_run[nt][rr] = bm[nt][rr];
                    l_part[nt][rr] *= alpha;
#pragma unroll
                    for (int mt = 0; mt < NK; ++mt) {
                        o[nt][mt][rr] *= alpha;
                        o[nt][mt][rr + 2] *= alpha;
                    }
                }
        }
        // ---- P = 2^(s - m); P^T fragments for the P.V MMA
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float m = m_run[nt][e & 1];
                pv[e] = s[nt][e] == -INFINITY ? 0.f : ex2(s[nt][e] - m);
                l_part[nt][e & 1] += pv[e];
            }
            pb[nt][0] = movmatrix_trans(pack2<T>(pv[0], pv[1]));   // keys 0-7 of the block
            pb[nt][1] = movmatrix_trans(pack2<T>(pv[2], pv[3]));   // keys 8-15
        }

        // ---- O^T += V^T P^T
#pragma unroll
        for (int mt = 0; mt < NK; ++mt) {
            uint32_t a[4];
            ldsm_x4_trans(sw128_addr(vs, kb + mrow + (mi >> 1) * 8, mt * 16 + (mi & 1) * 8), a);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_16816<T>(o[nt][mt], a, pb[nt][0], pb[nt][1]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars[NST + st]));
    }

    // ---- merge the warps of the CTA
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            float l = l_part[nt][rr];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            l_part[nt][rr] = l;
        }
    asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
    // every stage has been consumed (or the wait gave up): the ring is reused
    float* mo = reinterpret_cast<float*>(base_ptr);   // [NW][RM]
    float* lo = mo + NW * RM;                          // [NW][RM]
    float* oo = lo + NW * RM;                          // [NW][RM][D]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        if (lane < 4) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                mo[warp * RM + nt * 8 + rsub + rr] = m_run[nt][rr];
                lo[warp * RM + nt * 8 + rsub + rr] = l_part[nt][rr];
            }
        }
#pragma unroll
        for (int mt = 0; mt < NK; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = nt * 8 + rsub + (e & 1);
                const int dd = mt * 16 + lane / 4 + (e >> 1) * 8;
                oo[(warp * RM + r) * D + dd] = o[nt][mt][e];
            }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");

    const bool aborted = *abort_flag != 0;
    for (int idx = threadIdx.x; idx < p.Rv * D; idx += NW * 32) {
        const int r = idx / D, e = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, mo[w * RM + r]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = ex2(mo[w * RM + r] - M);
                L += f * lo[w * RM + r];
                acc += f * oo[(w * RM + r) * D + e];
            }
        }
        if (aborted) continue;
        if (p.nsplit == 1) {
            const int g = r / p.Tnew, t = r % p.Tnew;
            const size_t orow = (size_t(b) * p.H + size_t(kvh) * p.G + g) * p.Tnew + t;
            static_cast<T*>(p.o)[orow * D + e] = from_f32<T>(L > 0.f ? acc / L : 0.f);
            if (e == 0 && p.lse) p.lse[orow] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
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

}  // namespace b200attn
