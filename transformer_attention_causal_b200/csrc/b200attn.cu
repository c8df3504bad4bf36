// libb200attn: C-ABI entry points, argument checks, planning and launches.
// The operation, layouts, ownership and error rules are documented in
// include/b200attn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "b200attn.h"
#include "decode_splitkv.cuh"
#include "decode_mma.cuh"
#include "kv_append.cuh"
#include "prefill_backward.cuh"
#include "prefill_tcgen05.cuh"
#include "simt_attn.cuh"
#include "simt_backward.cuh"

using namespace b200attn;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<uint32_t> g_test_flags{0};

// Planning constant for B200: 148 SMs (the split plan fills the last wave of
// CTAs; the device's own count is read at launch where it matters).
constexpr int kPlanSMs = 148;

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }
size_t esize(attn_dtype_t dt) { return dt == ATTN_F32 ? 4 : 2; }

struct Problem {
    attn_dtype_t dt;
    int64_t B, H, Hkv, Tq, S, S_cap, d, start_pos;
    int causal;
    bool cached;  // attn_cached: split-KV decode allowed
    int64_t window = 0;  // local window (0: none); causal only
    bool paged = false;  // attn_cached_paged: K/V in page pools
};

struct Plan {
    attn_kernel_t kernel = ATTN_KERNEL_NONE;
    // split-KV decode
    int R = 0, Rv = 0, nsplit = 1;
    bool mma = false;    // warp-level MMA decode kernel (d = 64 or 128)
    int64_t chunk = 0, kv_end = 0, k_lo = 0;
    size_t ws_bytes = 0;
    // tcgen05 prefill
    int dch = 0, pair_mode = 0, n_qb = 0, units_per_level = 0, n_levels = 0, group = 1;
    int n_whole = 0, split = 1;   // units done whole; pieces per later unit
};

bool empty_problem(const Problem& pb) { return pb.B == 0 || pb.H == 0 || pb.Tq == 0; }

// Shape checks shared by every entry point (pointers are checked separately).
attn_status_t check_shape(const Problem& pb) {
    if (pb.dt != ATTN_F32 && pb.dt != ATTN_BF16 && pb.dt != ATTN_F16) return ATTN_ERR_INVALID_ARG;
    if (pb.B < 0 || pb.H < 0 || pb.Hkv < 0 || pb.Tq < 0 || pb.S < 0 || pb.S_cap < 0 ||
        pb.d < 0 || pb.start_pos < 0 || pb.window < 0 || (pb.window > 0 && !pb.causal))
        return ATTN_ERR_INVALID_ARG;
    if (empty_problem(pb)) return ATTN_OK;
    if (pb.Hkv == 0 || pb.H % pb.Hkv != 0 || pb.d == 0) return ATTN_ERR_INVALID_ARG;
    if (pb.S > pb.S_cap || pb.start_pos + pb.Tq > pb.S) return ATTN_ERR_INVALID_ARG;
    if (pb.d > kSimtMaxD) return ATTN_ERR_UNSUPPORTED;
    // 32-bit grid and index limits of the kernels
    if (pb.B * pb.H * pb.Tq > (int64_t(1) << 40) || pb.B * pb.Hkv > (int64_t(1) << 30))
        return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

int decode_rmax(int64_t d) {
    if (d % 16 == 0 && d >= 64 && d <= 128) return 16;
    if (d == 256) return 8;
    return 0;
}

int next_pow2_at_least4(int64_t x) {
    int r = 4;
    while (r < x) r <<= 1;
    return r;
}

void plan_decode(const Problem& pb, Plan& pl) {
    pl.kernel = ATTN_KERNEL_SPLITKV;
    const int64_t G = pb.H / pb.Hkv;
    pl.Rv = int(G * pb.Tq);
    pl.R = next_pow2_at_least4(pl.Rv);
    // d a multiple of 16 in [64, 128]: the MMA kernel (128-key stages, one CTA
    // per SM); d = 256: the CUDA-core kernel (64-key stages, two CTAs per SM)
    pl.mma = pb.d % 16 == 0 && pb.d >= 64 && pb.d <= 128 && pl.Rv <= 16;
    const int stage_keys = pl.mma ? kDecMmaTK : 64;
    const int ctas_per_sm = pl.mma ? 1 : 2;
    pl.kv_end = std::min<int64_t>(pb.S, pb.start_pos + pb.Tq);
    // a local window: no row sees a key below the first row's window
    pl.k_lo = pb.window > 0 ? std::max<int64_t>(0, pb.start_pos - pb.window + 1) : 0;
    const int64_t tiles = (pl.kv_end - pl.k_lo + stage_keys - 1) / stage_keys;
    const int64_t units = pb.B * pb.Hkv;
    const int64_t slots = int64_t(kPlanSMs) * ctas_per_sm;
    // Pick the split count with the least modelled time: waves of CTAs, each
    // costing its stages plus a start-up and merge worth about three stages
    // (one CTA per SM, so a wave's start is not hidden behind the last one's
    // stages); fewer splits on ties, at least 4 stages per split when there
    // is room.  Against filling the last wave best, this halves the CTAs of
    // mid-size calls (B = 8, S = 8192: 3.0 -> 3.9 TB/s at d = 96, 3.5 -> 4.3
    // at d = 128) and leaves the large ones as they were.
    int best_n = 1;
    double best_score = -1e300;
    const int64_t max_n = std::max<int64_t>(1, std::min<int64_t>(tiles, 128));
    for (int64_t n = 1; n <= max_n; ++n) {
        const int64_t per = (tiles + n - 1) / n;
        const int64_t n_eff = (tiles + per - 1) / per;  // no empty splits
        if (n_eff != n) continue;
        if (per < 4 && n > 1 && units * (n - 1) >= slots) continue;
        const int64_t ctas = units * n;
        const int64_t waves = (ctas + slots - 1) / slots;
        const double score = -double(waves) * (3.0 + double(per)) - 1e-3 * double(n);
        if (score > best_score + 1e-12) {
            best_score = score;
            best_n = int(n);
        }
    }
    const int64_t per = (tiles + best_n - 1) / best_n;
    pl.nsplit = best_n;
    pl.chunk = per * stage_keys;
    pl.ws_bytes = 0;
    if (pl.nsplit > 1) {
        const size_t rows = size_t(units) * pl.nsplit * pl.Rv;
        const size_t bytes = rows * size_t(pb.d + 2) * sizeof(float);
        pl.ws_bytes = (bytes + 255) & ~size_t(255);
    }
}

// Items per L2 group for grouped_order: whole runs of `per_run` items that
// share `run_bytes` of tiles, as many runs as fit kL2GroupBytes (a quarter
// of B200's 126 MB L2: the streams of Q and O pass through it too).
constexpr int64_t kL2GroupBytes = int64_t(32) << 20;
int l2_group(int64_t run_bytes, int64_t per_run, int64_t per_level) {
    const int64_t runs = std::max<int64_t>(1, kL2GroupBytes / std::max<int64_t>(run_bytes, 1));
    return int(std::max<int64_t>(1, std::min<int64_t>(runs * std::max<int64_t>(per_run, 1), per_level)));
}

// Key tiles of the first query tile's slot (the lightest units' range).
int64_t first_tile_keys(const Problem& pb) {
    const int64_t end = pb.causal ? std::min(pb.S, pb.start_pos + std::min<int64_t>(128, pb.Tq)) : pb.S;
    return (end + 127) / 128;
}

// Tail split of the tensor-core prefill (cached calls, no window): with U
// units on g CTAs (one per SM), the last pass holds R = U mod g units (all of
// them when U < g).  When R is at most half the CTAs, those units are cut into
// `split` pieces of at least 4 key tiles each (at most kMergeMaxSplit,
// R * split <= g), so the last pass costs about 1 / split of a unit instead of
// a whole one while the other CTAs would idle.  Only calls of at most 8 full
// passes, where that tail is worth the pieces' fp32 partials and the merge
// launch.  The pieces' workspace must fit `ws_cap` (fewer pieces otherwise).
void plan_tail_split(const Problem& pb, Plan& pl, size_t ws_cap) {
    pl.n_whole = pl.units_per_level * pl.n_levels;
    pl.split = 1;
    if (!pb.cached || pb.window > 0) return;
    const int64_t U = int64_t(pl.units_per_level) * pl.n_levels;
    const int64_t g = kPlanSMs;
    const int64_t full = U / g, R = U % g;
    if (R == 0 || 2 * R > g || full > 8) return;
    int64_t split = std::min<int64_t>(std::min<int64_t>(g / R, kMergeMaxSplit), first_tile_keys(pb) / 4);
    for (; split >= 2; --split) {
        const size_t bytes = size_t(R * split) * 2 * 128 * size_t(pb.d + 1) * sizeof(float);
        const size_t ws = (bytes + 255) & ~size_t(255);
        if (ws <= ws_cap) {
            pl.n_whole = int(full * g);
            pl.split = int(split);
            pl.ws_bytes = ws;
            return;
        }
    }
}

void plan_prefill_tc(const Problem& pb, Plan& pl, size_t ws_cap) {
    pl.kernel = ATTN_KERNEL_TCGEN05;
    const int64_t G = pb.H / pb.Hkv;
    pl.dch = pb.d <= 64 ? 1 : 2;
    pl.pair_mode = (G % 2 == 0) ? 0 : 1;
    pl.n_qb = int((pb.Tq + 127) / 128);
    if (pl.pair_mode == 0) {
        pl.units_per_level = int(pb.B * pb.Hkv * (G / 2));
        pl.n_levels = pl.n_qb;
    } else {
        pl.units_per_level = int(pb.B * pb.H);
        pl.n_levels = (pl.n_qb + 1) / 2;
    }
    // Level by level over every item (one group): grouping the items by the
    // L2 budget (l2_group) cut the GQA prefill's DRAM traffic from 2.8x to
    // 1.1x its algorithmic bytes but made it 6 % slower (every CTA in flight
    // then reads the same few K/V heads; DRAM was only ~30 % busy), so the
    // forward keeps the heaviest-first order across all items.
    pl.group = pl.units_per_level;
    plan_tail_split(pb, pl, ws_cap);
}

// `ws_cap`: the most workspace the call can be given (the no-allocation
// entry point's fixed array); plans that would need more use less.
attn_status_t make_plan(const Problem& pb, Plan& pl, size_t ws_cap = SIZE_MAX) {
    attn_status_t st = check_shape(pb);
    if (st != ATTN_OK) return st;
    pl = Plan();
    if (empty_problem(pb)) return ATTN_OK;
    if (pb.dt == ATTN_F32) {
        pl.kernel = ATTN_KERNEL_SIMT;
        return ATTN_OK;
    }
    const int64_t G = pb.H / pb.Hkv;
    const int rmax = decode_rmax(pb.d);
    if (pb.cached && rmax > 0 && G * pb.Tq <= rmax) {
        plan_decode(pb, pl);
        return ATTN_OK;
    }
    if (pb.d % 16 == 0 && pb.d >= 64 && pb.d <= 128 &&
        (pb.B * pb.Hkv * std::max<int64_t>(G / 2, 1) * ((pb.Tq + 127) / 128)) < (int64_t(1) << 31) &&
        pb.S_cap * pb.d * 2 < (int64_t(1) << 40)) {
        plan_prefill_tc(pb, pl, ws_cap);
        return ATTN_OK;
    }
    pl.kernel = ATTN_KERNEL_SIMT;
    return ATTN_OK;
}

// ------------------------------------------------------------------ TMA maps

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

attn_status_t get_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? ATTN_OK : ATTN_ERR_CUDA;
}

// [nslices, rows (pitch row_pitch), d] 16-bit tensor, box of 64 columns x
// box_rows rows (128 unless a paged pool's pages are smaller).
attn_status_t encode_rows(CUtensorMap* map, const void* ptr, attn_dtype_t dt, int64_t d,
                          int64_t rows, int64_t row_pitch, int64_t nslices, uint32_t box_rows = 128) {
    const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(rows), cuuint64_t(nslices)};
    const cuuint64_t strides[2] = {cuuint64_t(d * 2), cuuint64_t(row_pitch * d * 2)};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType ty =
        dt == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = g_encode(map, ty, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// ------------------------------------------------------------------ launches

template <typename K>
attn_status_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) ==
                   cudaSuccess
               ? ATTN_OK
               : ATTN_ERR_CUDA;
}

constexpr int kMaxDevices = 64;

// Once per kernel and device: its dynamic shared-memory limit and, for a
// kernel that moves registers between warpgroups (setmaxnreg), a check that
// its launch allocation (threads x registers) covers `regs_needed`, since an
// increase the block's pool cannot grant never returns.  The outcome is kept
// and returned on every later call, so a failure is never followed by a
// launch.
template <auto Kern>
attn_status_t prepare_kernel(size_t smem, int threads = 0, int regs_needed = 0) {
    static std::once_flag once[kMaxDevices];
    static attn_status_t status[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::call_once(once[dev], [&] {
        attn_status_t r = set_smem(Kern, smem);
        if (r == ATTN_OK && regs_needed > 0) {
            cudaFuncAttributes fa{};
            if (cudaFuncGetAttributes(&fa, Kern) != cudaSuccess || fa.numRegs * threads < regs_needed)
                r = ATTN_ERR_CUDA;
        }
        status[dev] = r;
    });
    return status[dev];
}

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kPlanSMs;
    int n = cached[dev].load();
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = kPlanSMs;
        cached[dev].store(n);
    }
    return n;
}

attn_status_t launch_status() {
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename T>
attn_status_t run_simt(const Problem& pb, const void* q, const void* k, const void* v, void* o,
                       float* lse, float scale, cudaStream_t stream) {
    SimtParams sp;
    sp.q = q; sp.k = k; sp.v = v; sp.o = o; sp.lse = lse;
    sp.B = pb.B; sp.H = pb.H; sp.Hkv = pb.Hkv; sp.Tq = pb.Tq; sp.S = pb.S; sp.S_cap = pb.S_cap;
    sp.d = pb.d; sp.start_pos = pb.start_pos; sp.scale = scale; sp.causal = pb.causal;
    sp.window = pb.window;
    const int64_t rows = pb.B * pb.H * pb.Tq;
    const int64_t blocks = (rows + kSimtWarps - 1) / kSimtWarps;
    if (blocks > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    simt_attention_kernel<T><<<unsigned(blocks), kSimtWarps * 32, 0, stream>>>(sp);
    return launch_status();
}

// The split merge, launched as a programmatic dependent of the decode kernel
// just enqueued on `stream`: its launch overlaps the decode's tail and it
// waits (griddepcontrol.wait) for the decode grid's results.
template <typename T, int D>
attn_status_t launch_combine(const DecodeParams& dp, cudaStream_t stream) {
    const int64_t rows = int64_t(dp.B) * dp.Hkv * dp.Rv;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(unsigned((rows + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel<T, D>, dp) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename T, int D, int R, int MODE>
attn_status_t launch_decode_RP(const DecodeParams& dp, cudaStream_t stream) {
    constexpr size_t smem = DecodeShape<D, R>::smem_bytes(sizeof(T));
    constexpr auto kern = &decode_splitkv_kernel<T, D, R, MODE>;
    if (const attn_status_t st = prepare_kernel<kern>(smem); st != ATTN_OK) return st;
    dim3 grid(unsigned(dp.nsplit), unsigned(dp.B * dp.Hkv));
    kern<<<grid, 160, smem, stream>>>(dp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_CUDA;
    if (dp.nsplit > 1) return launch_combine<T, D>(dp, stream);
    return ATTN_OK;
}

template <typename T, int D, int R>
attn_status_t launch_decode_R(const DecodeParams& dp, cudaStream_t stream) {
    if (dp.paged) return launch_decode_RP<T, D, R, kDecodePaged>(dp, stream);
    if (dp.window > 0) return launch_decode_RP<T, D, R, kDecodeWindow>(dp, stream);
    return launch_decode_RP<T, D, R, kDecodePlain>(dp, stream);
}

// The CUDA-core split-KV decode (d = 256; R = G * Tnew padded to 4 or 8).
template <typename T>
attn_status_t launch_decode_256(int R, const DecodeParams& dp, cudaStream_t stream) {
    switch (R) {
    case 4: return launch_decode_R<T, 256, 4>(dp, stream);
    case 8: return launch_decode_R<T, 256, 8>(dp, stream);
    default: return ATTN_ERR_UNSUPPORTED;
    }
}

template <typename T, int D, int NT, bool WINDOW, bool PAGED = false>
attn_status_t launch_decode_mma_k(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& dp,
                                  cudaStream_t stream) {
    constexpr size_t smem = DecMmaShape<(D + 63) / 64>::smem_bytes();
    constexpr auto kern = &decode_mma_kernel<T, D, NT, WINDOW, PAGED>;
    if (const attn_status_t st = prepare_kernel<kern>(smem); st != ATTN_OK) return st;
    dim3 grid(unsigned(dp.nsplit), unsigned(dp.B * dp.Hkv));
    kern<<<grid, kDecMmaThreads, smem, stream>>>(mk, mv, dp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_CUDA;
    if (dp.nsplit > 1) return launch_combine<T, D>(dp, stream);
    return ATTN_OK;
}

// One head size: rows padded to 8 or 16; plain, windowed or paged cache.
template <typename T, int D>
attn_status_t launch_decode_mma_d(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& dp,
                                  cudaStream_t stream) {
    const bool two = dp.Rv > 8;
    if (dp.paged)
        return two ? launch_decode_mma_k<T, D, 2, false, true>(mk, mv, dp, stream)
                   : launch_decode_mma_k<T, D, 1, false, true>(mk, mv, dp, stream);
    if (dp.window > 0)
        return two ? launch_decode_mma_k<T, D, 2, true>(mk, mv, dp, stream)
                   : launch_decode_mma_k<T, D, 1, true>(mk, mv, dp, stream);
    return two ? launch_decode_mma_k<T, D, 2, false>(mk, mv, dp, stream)
               : launch_decode_mma_k<T, D, 1, false>(mk, mv, dp, stream);
}

template <typename T>
attn_status_t launch_decode_mma(const Problem& pb, const DecodeParams& dp, cudaStream_t stream,
                                int64_t page_size = 0) {
    if (get_encoder() != ATTN_OK) return ATTN_ERR_CUDA;
    CUtensorMap mk, mv;
    if (dp.paged) {
        // the page pools as [num_pages * Hkv, P, d], boxes of min(P, 128) rows
        const uint32_t rows = uint32_t(std::min<int64_t>(page_size, kDecMmaTK));
        if (encode_rows(&mk, dp.k, pb.dt, pb.d, page_size, page_size, dp.num_pages * pb.Hkv, rows) != ATTN_OK ||
            encode_rows(&mv, dp.v, pb.dt, pb.d, page_size, page_size, dp.num_pages * pb.Hkv, rows) != ATTN_OK)
            return ATTN_ERR_CUDA;
    } else if (encode_rows(&mk, dp.k, pb.dt, pb.d, pb.S, pb.S_cap, pb.B * pb.Hkv) != ATTN_OK ||
               encode_rows(&mv, dp.v, pb.dt, pb.d, pb.S, pb.S_cap, pb.B * pb.Hkv) != ATTN_OK) {
        return ATTN_ERR_CUDA;
    }
    switch (pb.d) {
    case 64: return launch_decode_mma_d<T, 64>(mk, mv, dp, stream);
    case 80: return launch_decode_mma_d<T, 80>(mk, mv, dp, stream);
    case 96: return launch_decode_mma_d<T, 96>(mk, mv, dp, stream);
    case 112: return launch_decode_mma_d<T, 112>(mk, mv, dp, stream);
    case 128: return launch_decode_mma_d<T, 128>(mk, mv, dp, stream);
    default: return ATTN_ERR_UNSUPPORTED;
    }
}

// A paged K/V cache: page pools, the page table and the per-sequence lengths.
struct PagedKV {
    const int32_t* page_table = nullptr;
    const int32_t* kv_lens = nullptr;
    int64_t max_pages = 0, num_pages = 0;
    int page_shift = 0;
};

template <typename T>
attn_status_t run_decode(const Problem& pb, const Plan& pl, const void* q, const void* k,
                         const void* v, void* o, float* lse, float scale, void* ws,
                         cudaStream_t stream, const PagedKV* paged = nullptr) {
    DecodeParams dp{};
    dp.q = q; dp.k = k; dp.v = v; dp.o = o; dp.lse = lse;
    const size_t rows = size_t(pb.B * pb.Hkv) * pl.nsplit * pl.Rv;
    float* wsf = static_cast<float*>(ws);
    dp.ws_o = wsf;
    dp.ws_m = wsf ? wsf + rows * pb.d : nullptr;
    dp.ws_l = wsf ? dp.ws_m + rows : nullptr;
    dp.B = int(pb.B); dp.H = int(pb.H); dp.Hkv = int(pb.Hkv);
    dp.G = int(pb.H / pb.Hkv); dp.Tnew = int(pb.Tq); dp.Rv = pl.Rv;
    dp.S = pb.S; dp.S_cap = pb.S_cap; dp.start_pos = pb.start_pos;
    dp.kv_end = pl.kv_end; dp.chunk = pl.chunk; dp.nsplit = pl.nsplit;
    dp.k_lo = pl.k_lo; dp.window = pb.window;
    dp.scale_log2 = scale * 1.4426950408889634f;
    dp.timeout_ns = g_timeout_ns.load();
    dp.test_flags = g_test_flags.load();
    if (paged) {
        dp.paged = 1;
        dp.page_shift = paged->page_shift;
        dp.page_table = paged->page_table;
        dp.kv_lens = paged->kv_lens;
        dp.max_pages = paged->max_pages;
        dp.num_pages = paged->num_pages;
    }
    if (pl.mma) return launch_decode_mma<T>(pb, dp, stream, paged ? (int64_t(1) << paged->page_shift) : 0);
    if (pb.d == 256) return launch_decode_256<T>(pl.R, dp, stream);
    return ATTN_ERR_UNSUPPORTED;
}

template <typename T, int DCH, bool WINDOW, bool PAGED, bool SPLIT>
attn_status_t launch_prefill_kernel(const CUtensorMap& mq, const CUtensorMap& mk,
                                    const CUtensorMap& mv, const PrefillParams& pp, int64_t grid,
                                    cudaStream_t stream) {
    constexpr size_t smem = prefill_smem_bytes<DCH>();
    constexpr auto kern = &prefill_tcgen05_kernel<T, DCH, WINDOW, PAGED, SPLIT>;
    // the register split: warpgroup 0 at kPfRegsLow, the two softmax warpgroups at kPfRegsHigh
    if (const attn_status_t st =
            prepare_kernel<kern>(smem, kPfThreads, 128 * kPfRegsLow + 256 * kPfRegsHigh);
        st != ATTN_OK)
        return st;
    kern<<<unsigned(grid), kPfThreads, smem, stream>>>(mq, mk, mv, pp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_CUDA;
    if (pp.split <= 1) return ATTN_OK;
    // the pieces' merge, as a programmatic dependent (as the decode's
    // combine): one warp per row, 256 rows per split unit
    const int64_t rows = int64_t(pp.units_per_level * pp.n_levels - pp.n_whole) * 256;
    const int64_t warps_per_block = kMergeThreads / 32;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(unsigned((rows + warps_per_block - 1) / warps_per_block));
    cfg.blockDim = dim3(kMergeThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_merge_kernel<T>, pp) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Work items of a plan and the pieces' workspace.
void set_items(PrefillParams& pp, const Plan& pl, const Problem& pb, void* ws) {
    pp.n_whole = pl.n_whole;
    pp.split = pl.split;
    pp.ws_o = nullptr;
    pp.ws_lse = nullptr;
    if (pl.split > 1) {
        const size_t rows = size_t(pl.units_per_level * pl.n_levels - pl.n_whole) * pl.split * 256;
        pp.ws_o = static_cast<float*>(ws);
        pp.ws_lse = pp.ws_o + rows * size_t(pb.d);
    }
}

template <typename T, int DCH>
attn_status_t launch_prefill_tc(const Problem& pb, const Plan& pl, const void* q, const void* k,
                                const void* v, void* o, float* lse, float scale, void* ws,
                                cudaStream_t stream) {
    if (get_encoder() != ATTN_OK) return ATTN_ERR_CUDA;
    CUtensorMap mq, mk, mv;
    if (encode_rows(&mq, q, pb.dt, pb.d, pb.Tq, pb.Tq, pb.B * pb.H) != ATTN_OK ||
        encode_rows(&mk, k, pb.dt, pb.d, pb.S, pb.S_cap, pb.B * pb.Hkv) != ATTN_OK ||
        encode_rows(&mv, v, pb.dt, pb.d, pb.S, pb.S_cap, pb.B * pb.Hkv) != ATTN_OK)
        return ATTN_ERR_CUDA;
    PrefillParams pp{};
    pp.o = o; pp.lse = lse;
    pp.B = int(pb.B); pp.H = int(pb.H); pp.Hkv = int(pb.Hkv); pp.G = int(pb.H / pb.Hkv);
    pp.Tq = int(pb.Tq); pp.S = pb.S; pp.start_pos = pb.start_pos; pp.d = int(pb.d);
    pp.causal = pb.causal; pp.pair_mode = pl.pair_mode; pp.n_qb = pl.n_qb;
    pp.window = pb.window;
    pp.units_per_level = pl.units_per_level;
    pp.n_levels = pl.n_levels;
    pp.group = pl.group;
    pp.scale_log2 = scale == 0.f ? 1.f : std::fabs(scale) * 1.4426950408889634f;
    pp.score_mode = scale > 0.f ? 0 : (scale < 0.f ? 1 : 2);
    pp.timeout_ns = g_timeout_ns.load();
    pp.test_flags = g_test_flags.load();
    set_items(pp, pl, pb, ws);
    // persistent CTAs, one per SM (the kernel deals the work items out itself)
    const int64_t grid = std::min<int64_t>(prefill_items(pp), sm_count());
    // pieces only in cached calls without a window (plan_tail_split)
    if (pb.window > 0) return launch_prefill_kernel<T, DCH, true, false, false>(mq, mk, mv, pp, grid, stream);
    return pp.split > 1 ? launch_prefill_kernel<T, DCH, false, false, true>(mq, mk, mv, pp, grid, stream)
                        : launch_prefill_kernel<T, DCH, false, false, false>(mq, mk, mv, pp, grid, stream);
}

// The tensor-core prefill over a paged cache (chunked prefill): K/V maps over
// the pools [num_pages * Hkv, P, d] with boxes of min(P, 128) rows.
template <typename T, int DCH>
attn_status_t launch_prefill_paged(const Problem& pb, const Plan& pl, const void* q, const void* kp,
                                   const void* vp, void* o, float* lse, float scale,
                                   const PagedKV& pk, int64_t page_size, void* ws, cudaStream_t stream) {
    if (get_encoder() != ATTN_OK) return ATTN_ERR_CUDA;
    CUtensorMap mq, mk, mv;
    const uint32_t rows = uint32_t(std::min<int64_t>(page_size, 128));
    if (encode_rows(&mq, q, pb.dt, pb.d, pb.Tq, pb.Tq, pb.B * pb.H) != ATTN_OK ||
        encode_rows(&mk, kp, pb.dt, pb.d, page_size, page_size, pk.num_pages * pb.Hkv, rows) != ATTN_OK ||
        encode_rows(&mv, vp, pb.dt, pb.d, page_size, page_size, pk.num_pages * pb.Hkv, rows) != ATTN_OK)
        return ATTN_ERR_CUDA;
    PrefillParams pp{};
    pp.o = o; pp.lse = lse;
    pp.B = int(pb.B); pp.H = int(pb.H); pp.Hkv = int(pb.Hkv); pp.G = int(pb.H / pb.Hkv);
    pp.Tq = int(pb.Tq); pp.S = pb.S; pp.start_pos = pb.start_pos; pp.d = int(pb.d);
    pp.causal = 1; pp.pair_mode = pl.pair_mode; pp.n_qb = pl.n_qb;
    pp.window = 0;
    pp.units_per_level = pl.units_per_level;
    pp.n_levels = pl.n_levels;
    pp.group = pl.group;
    pp.scale_log2 = scale == 0.f ? 1.f : std::fabs(scale) * 1.4426950408889634f;
    pp.score_mode = scale > 0.f ? 0 : (scale < 0.f ? 1 : 2);
    pp.timeout_ns = g_timeout_ns.load();
    pp.test_flags = g_test_flags.load();
    pp.page_table = pk.page_table;
    pp.kv_lens = pk.kv_lens;
    pp.max_pages = pk.max_pages;
    pp.num_pages = pk.num_pages;
    pp.max_kv_len = pb.S;
    pp.page_shift = pk.page_shift;
    set_items(pp, pl, pb, ws);
    const int64_t grid = std::min<int64_t>(prefill_items(pp), sm_count());
    return pp.split > 1 ? launch_prefill_kernel<T, DCH, false, true, true>(mq, mk, mv, pp, grid, stream)
                        : launch_prefill_kernel<T, DCH, false, true, false>(mq, mk, mv, pp, grid, stream);
}

template <typename T>
attn_status_t run_prefill_tc(const Problem& pb, const Plan& pl, const void* q, const void* k,
                             const void* v, void* o, float* lse, float scale, void* ws,
                             cudaStream_t stream) {
    if (pl.dch == 1) return launch_prefill_tc<T, 1>(pb, pl, q, k, v, o, lse, scale, ws, stream);
    return launch_prefill_tc<T, 2>(pb, pl, q, k, v, o, lse, scale, ws, stream);
}

attn_status_t dispatch(const Problem& pb, const Plan& pl, const void* q, const void* k,
                       const void* v, void* o, float* lse, float scale, void* ws,
                       cudaStream_t stream) {
    switch (pl.kernel) {
    case ATTN_KERNEL_NONE: return ATTN_OK;
    case ATTN_KERNEL_SIMT:
        if (pb.dt == ATTN_F32) return run_simt<float>(pb, q, k, v, o, lse, scale, stream);
        if (pb.dt == ATTN_BF16) return run_simt<__nv_bfloat16>(pb, q, k, v, o, lse, scale, stream);
        return run_simt<__half>(pb, q, k, v, o, lse, scale, stream);
    case ATTN_KERNEL_SPLITKV:
        if (pb.dt == ATTN_BF16)
            return run_decode<__nv_bfloat16>(pb, pl, q, k, v, o, lse, scale, ws, stream);
        return run_decode<__half>(pb, pl, q, k, v, o, lse, scale, ws, stream);
    case ATTN_KERNEL_TCGEN05:
        if (pb.dt == ATTN_BF16)
            return run_prefill_tc<__nv_bfloat16>(pb, pl, q, k, v, o, lse, scale, ws, stream);
        return run_prefill_tc<__half>(pb, pl, q, k, v, o, lse, scale, ws, stream);
    }
    return ATTN_ERR_INVALID_ARG;
}

attn_status_t check_pointers(const Problem& pb, const void* q, const void* k, const void* v,
                             const void* o, const float* lse) {
    if (empty_problem(pb)) return ATTN_OK;
    if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if (lse && !aligned4(lse)) return ATTN_ERR_INVALID_ARG;
    return ATTN_OK;
}

}  // namespace

namespace {

template <typename T, int KB>
attn_status_t run_append(const AppendParams& ap, int threads, cudaStream_t stream) {
    const int64_t groups = (int64_t(ap.Tnew) + ap.tok_per_cta - 1) / ap.tok_per_cta;
    const int64_t blocks = int64_t(ap.B) * groups;
    if (blocks > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    kv_append_rope_kernel<T, KB><<<unsigned(blocks), threads, 0, stream>>>(ap);
    return launch_status();
}

template <typename T>
attn_status_t launch_append(AppendParams& ap, cudaStream_t stream) {
    const int esz = int(sizeof(T));
    const int half_bytes = ap.d / 2 * esz;
    const int kb = half_bytes % 16 == 0 ? 16 : 8;   // d/2 * esz is a multiple of 8
    ap.half_units = half_bytes / kb;
    const int per_tok = 2 * ap.Hkv * ap.half_units;
    ap.div_tok = FastDiv(uint32_t(per_tok));
    ap.div_row = FastDiv(uint32_t(ap.half_units));
    const int threads = std::min(256, (per_tok + 31) / 32 * 32);
    // as many tokens as fill every thread's units, at most kAppendMaxTok
    ap.tok_per_cta = std::max(1, std::min(std::min(kAppendMaxTok, ap.Tnew),
                                          threads * kAppendUnits / per_tok));
    return kb == 16 ? run_append<T, 16>(ap, threads, stream) : run_append<T, 8>(ap, threads, stream);
}

}  // namespace

namespace {

// The tensor-core backward kernels take 16-bit inputs with d a multiple of
// 16 in [64, 128]; everything else up to d = 256 runs on CUDA cores.
bool backward_on_tensor_cores(const Problem& pb) {
    return pb.dt != ATTN_F32 && pb.d % 16 == 0 && pb.d >= 64 && pb.d <= 128;
}

attn_status_t check_backward(const Problem& pb) {
    attn_status_t st = check_shape(pb);
    if (st != ATTN_OK || empty_problem(pb)) return st;
    const int64_t n_t = (pb.Tq + 127) / 128;
    const int64_t rows = std::max(pb.B * pb.H, pb.B * pb.Hkv) * n_t * 128;
    if (n_t * pb.B * pb.H >= (int64_t(1) << 31) || pb.Tq >= (int64_t(1) << 30) ||
        rows / kSimtBwdWarps >= (int64_t(1) << 31) || pb.S_cap * pb.d * 2 >= (int64_t(1) << 40))
        return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

template <typename T>
attn_status_t launch_backward_simt(BwdParams& bp, const void* q, const void* k, const void* v,
                                   cudaStream_t stream) {
    const SimtBwdPtrs in{q, k, v};
    const auto blocks = [](int64_t rows) { return unsigned((rows + kSimtBwdWarps - 1) / kSimtBwdWarps); };
    simt_bwd_preprocess_kernel<T><<<blocks(int64_t(bp.B) * bp.H * bp.Tpad), kSimtBwdWarps * 32, 0,
                                    stream>>>(bp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_CUDA;
    simt_bwd_dkdv_kernel<T><<<blocks(int64_t(bp.B) * bp.Hkv * bp.T), kSimtBwdWarps * 32, 0, stream>>>(
        bp, in);
    if (launch_status() != ATTN_OK) return ATTN_ERR_CUDA;
    simt_bwd_dq_kernel<T><<<blocks(int64_t(bp.B) * bp.H * bp.T), kSimtBwdWarps * 32, 0, stream>>>(bp, in);
    return launch_status();
}

size_t backward_ws_bytes(const Problem& pb) {
    const int64_t tpad = (pb.Tq + 127) / 128 * 128;
    const size_t bytes = size_t(2) * size_t(pb.B * pb.H * tpad) * sizeof(float);
    return (bytes + 255) & ~size_t(255);
}

template <typename T, int DCH, bool WINDOW>
attn_status_t launch_backward(const Problem& pb, BwdParams& bp, const void* q, const void* k,
                              const void* v, const void* dout, cudaStream_t stream) {
    if (get_encoder() != ATTN_OK) return ATTN_ERR_CUDA;
    CUtensorMap mq, mk, mv, mdo;
    if (encode_rows(&mq, q, pb.dt, pb.d, pb.Tq, pb.Tq, pb.B * pb.H) != ATTN_OK ||
        encode_rows(&mdo, dout, pb.dt, pb.d, pb.Tq, pb.Tq, pb.B * pb.H) != ATTN_OK ||
        encode_rows(&mk, k, pb.dt, pb.d, pb.S, pb.S_cap, pb.B * pb.Hkv) != ATTN_OK ||
        encode_rows(&mv, v, pb.dt, pb.d, pb.S, pb.S_cap, pb.B * pb.Hkv) != ATTN_OK)
        return ATTN_ERR_CUDA;
    const int64_t rows = int64_t(bp.B) * bp.H * bp.Tpad;
    const int64_t pre_blocks = std::min<int64_t>((rows + 15) / 16, int64_t(sm_count()) * 16);
    bwd_preprocess_kernel<T><<<unsigned(pre_blocks), 256, 0, stream>>>(bp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_CUDA;

    constexpr size_t smem_kv = bwd_dkdv_smem_bytes<DCH>();
    constexpr size_t smem_q = bwd_dq_smem_bytes<DCH>();
    constexpr auto kern_kv = &bwd_dkdv_kernel<T, DCH, WINDOW>;
    constexpr auto kern_q = &bwd_dq_kernel<T, DCH, WINDOW>;
    if (prepare_kernel<kern_kv>(smem_kv) != ATTN_OK || prepare_kernel<kern_q>(smem_q) != ATTN_OK)
        return ATTN_ERR_CUDA;
    kern_kv<<<unsigned(int64_t(bp.n_t) * bp.B * bp.Hkv), kBwdThreads, smem_kv, stream>>>(mq, mk, mv,
                                                                                        mdo, bp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_CUDA;
    kern_q<<<unsigned(int64_t(bp.n_t) * bp.B * bp.H), kBwdThreads, smem_q, stream>>>(mq, mk, mv, mdo,
                                                                                    bp);
    return launch_status();
}

}  // namespace

extern "C" {

attn_status_t attn_kv_append_rope(const void* k_new, const void* v_new, void* k_cache,
                                  void* v_cache, attn_dtype_t dtype, int64_t B, int64_t Hkv,
                                  int64_t Tnew, int64_t S_cap, int64_t d, int64_t start_pos,
                                  float rope_base, void* stream) {
    if (dtype != ATTN_F32 && dtype != ATTN_BF16 && dtype != ATTN_F16) return ATTN_ERR_INVALID_ARG;
    if (B < 0 || Hkv < 0 || Tnew < 0 || S_cap < 0 || d < 0 || start_pos < 0)
        return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(rope_base)) return ATTN_ERR_INVALID_ARG;
    if (B == 0 || Hkv == 0 || Tnew == 0) return ATTN_OK;
    const int64_t dmult = dtype == ATTN_F32 ? 4 : 8;
    if (d == 0 || d % dmult != 0) return ATTN_ERR_INVALID_ARG;
    if (d > kAppendMaxD) return ATTN_ERR_UNSUPPORTED;
    if (start_pos + Tnew > S_cap) return ATTN_ERR_INVALID_ARG;
    if (!k_new || !v_new || !k_cache || !v_cache) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return ATTN_ERR_INVALID_ARG;
    if (B * Tnew > (int64_t(1) << 31) || Hkv > (int64_t(1) << 16)) return ATTN_ERR_UNSUPPORTED;
    AppendParams ap{};
    ap.k_new = k_new; ap.v_new = v_new; ap.k_cache = k_cache; ap.v_cache = v_cache;
    ap.B = int(B); ap.Hkv = int(Hkv); ap.Tnew = int(Tnew); ap.d = int(d);
    ap.S_cap = S_cap; ap.start_pos = start_pos;
    ap.rotate = rope_base > 0.f ? 1 : 0;
    // inverse frequencies base^(-2i/d), formed in double on the host
    for (int64_t i = 0; ap.rotate && i < d / 2; ++i)
        ap.inv_freq[i] = std::pow(double(rope_base), -2.0 * double(i) / double(d));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == ATTN_F32) return launch_append<float>(ap, s);
    if (dtype == ATTN_BF16) return launch_append<__nv_bfloat16>(ap, s);
    return launch_append<__half>(ap, s);
}

attn_status_t attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                           attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv, int64_t T,
                           int64_t d, float scale, int causal, void* stream) {
    Problem pb{dtype, B, H, Hkv, T, T, T, d, 0, causal ? 1 : 0, false};
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    Plan pl;
    attn_status_t st = make_plan(pb, pl);
    if (st != ATTN_OK) return st;
    st = check_pointers(pb, q, k, v, o, lse);
    if (st != ATTN_OK) return st;
    return dispatch(pb, pl, q, k, v, o, lse, scale, nullptr, static_cast<cudaStream_t>(stream));
}

size_t attn_prefill_backward_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                                            int64_t T, int64_t d) {
    Problem pb{dtype, B, H, Hkv, T, T, T, d, 0, 1, false};
    if (check_backward(pb) != ATTN_OK || empty_problem(pb)) return 0;
    return backward_ws_bytes(pb);
}

}  // extern "C"

namespace {

attn_status_t prefill_backward(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv,
                               attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv, int64_t T,
                               int64_t d, float scale, int causal, int64_t window, void* workspace,
                               size_t workspace_bytes, void* stream) {
    Problem pb{dtype, B, H, Hkv, T, T, T, d, 0, causal ? 1 : 0, false, window};
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    attn_status_t st = check_backward(pb);
    if (st != ATTN_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (empty_problem(pb)) {
        // no query head reads the keys: their gradients are zero
        const size_t kv_bytes = size_t(B * Hkv * T * d) * esize(dtype);
        if (kv_bytes == 0) return ATTN_OK;
        if (!dk || !dv) return ATTN_ERR_INVALID_ARG;
        return cudaMemsetAsync(dk, 0, kv_bytes, s) == cudaSuccess &&
                       cudaMemsetAsync(dv, 0, kv_bytes, s) == cudaSuccess
                   ? ATTN_OK
                   : ATTN_ERR_CUDA;
    }
    const void* bufs[8] = {q, k, v, o, dout, dq, dk, dv};
    for (const void* ptr : bufs)
        if (!ptr || !aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
    if (!lse || !aligned4(lse)) return ATTN_ERR_INVALID_ARG;
    const size_t need = backward_ws_bytes(pb);
    if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
    BwdParams bp;
    bp.o = o; bp.dout = dout; bp.lse = lse;
    bp.dq = dq; bp.dk = dk; bp.dv = dv;
    bp.B = int(B); bp.H = int(H); bp.Hkv = int(Hkv); bp.G = int(H / Hkv); bp.T = int(T);
    bp.n_t = int((T + 127) / 128);
    // dK/dV: a (b, K/V head) streams the Q and dO tiles of its G heads;
    // dQ: a (b, head) streams its K/V head's tiles, shared by G heads
    bp.group_kv = l2_group(H / Hkv * T * d * 2 * 2, 1, B * Hkv);
    bp.group_q = l2_group(T * d * 2 * 2, H / Hkv, B * H);
    bp.Tpad = bp.n_t * 128;
    bp.d = int(d); bp.causal = causal ? 1 : 0;
    // a window covering every key is plain causal attention
    bp.window = (window > 0 && window < T) ? int(window) : 0;
    bp.nl = static_cast<float*>(workspace);
    bp.dd = bp.nl + size_t(B * H) * bp.Tpad;
    bp.scale = scale;
    bp.scale_log2 = scale * 1.4426950408889634f;
    bp.timeout_ns = g_timeout_ns.load();
    bp.test_flags = g_test_flags.load();
    const bool bf16 = dtype == ATTN_BF16;
    if (!backward_on_tensor_cores(pb)) {
        if (dtype == ATTN_F32) return launch_backward_simt<float>(bp, q, k, v, s);
        return bf16 ? launch_backward_simt<__nv_bfloat16>(bp, q, k, v, s)
                    : launch_backward_simt<__half>(bp, q, k, v, s);
    }
    if (bp.window > 0) {
        if (d <= 64)
            return bf16 ? launch_backward<__nv_bfloat16, 1, true>(pb, bp, q, k, v, dout, s)
                        : launch_backward<__half, 1, true>(pb, bp, q, k, v, dout, s);
        return bf16 ? launch_backward<__nv_bfloat16, 2, true>(pb, bp, q, k, v, dout, s)
                    : launch_backward<__half, 2, true>(pb, bp, q, k, v, dout, s);
    }
    if (d <= 64)
        return bf16 ? launch_backward<__nv_bfloat16, 1, false>(pb, bp, q, k, v, dout, s)
                    : launch_backward<__half, 1, false>(pb, bp, q, k, v, dout, s);
    return bf16 ? launch_backward<__nv_bfloat16, 2, false>(pb, bp, q, k, v, dout, s)
                : launch_backward<__half, 2, false>(pb, bp, q, k, v, dout, s);
}

}  // namespace

extern "C" {

attn_status_t attn_prefill_backward(const void* q, const void* k, const void* v, const void* o,
                                    const float* lse, const void* dout, void* dq, void* dk,
                                    void* dv, attn_dtype_t dtype, int64_t B, int64_t H,
                                    int64_t Hkv, int64_t T, int64_t d, float scale, int causal,
                                    void* workspace, size_t workspace_bytes, void* stream) {
    return prefill_backward(q, k, v, o, lse, dout, dq, dk, dv, dtype, B, H, Hkv, T, d, scale, causal, 0,
                            workspace, workspace_bytes, stream);
}

attn_status_t attn_prefill_backward_local(const void* q, const void* k, const void* v, const void* o,
                                          const float* lse, const void* dout, void* dq, void* dk,
                                          void* dv, attn_dtype_t dtype, int64_t B, int64_t H,
                                          int64_t Hkv, int64_t T, int64_t d, float scale,
                                          int64_t window, void* workspace, size_t workspace_bytes,
                                          void* stream) {
    return prefill_backward(q, k, v, o, lse, dout, dq, dk, dv, dtype, B, H, Hkv, T, d, scale, 1, window,
                            workspace, workspace_bytes, stream);
}

attn_status_t attn_cached(const void* q, const void* k_hist, const void* v_hist, void* o,
                          float* lse, attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                          int64_t Tnew, int64_t S, int64_t S_cap, int64_t d, int64_t start_pos,
                          float scale, void* workspace, size_t workspace_bytes, void* stream) {
    Problem pb{dtype, B, H, Hkv, Tnew, S, S_cap, d, start_pos, 1, true};
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    Plan pl;
    attn_status_t st = make_plan(pb, pl);
    if (st != ATTN_OK) return st;
    st = check_pointers(pb, q, k_hist, v_hist, o, lse);
    if (st != ATTN_OK) return st;
    if (pl.ws_bytes > 0) {
        if (!workspace || workspace_bytes < pl.ws_bytes) return ATTN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
    }
    return dispatch(pb, pl, q, k_hist, v_hist, o, lse, scale, workspace,
                    static_cast<cudaStream_t>(stream));
}

namespace {

// The problem a paged call plans as: every sequence at the host's length bound.
Problem paged_problem(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv, int64_t Tnew,
                      int64_t d, int64_t max_kv_len) {
    return Problem{dtype, B, H, Hkv, Tnew, max_kv_len, max_kv_len, d,
                   max_kv_len - Tnew, 1, true, 0, true};
}

}  // namespace

attn_status_t attn_cached_paged(const void* q, const void* k_pages, const void* v_pages, void* o,
                                float* lse, attn_dtype_t dtype, int64_t B, int64_t H,
                                int64_t Hkv, int64_t Tnew, int64_t d, const int32_t* page_table,
                                int64_t max_pages, int64_t num_pages, int64_t page_size,
                                const int32_t* kv_lens, int64_t max_kv_len, float scale,
                                void* workspace, size_t workspace_bytes, void* stream) {
    if (!std::isfinite(scale) || max_kv_len < 0 || max_pages < 0 || num_pages < 0 || page_size < 0)
        return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_F16) {
        if (dtype == ATTN_F32) return ATTN_ERR_UNSUPPORTED;
        return ATTN_ERR_INVALID_ARG;
    }
    if (B < 0 || H < 0 || Hkv < 0 || Tnew < 0 || d < 0) return ATTN_ERR_INVALID_ARG;
    if (B == 0 || H == 0 || Tnew == 0) return ATTN_OK;
    if (page_size < 8 || page_size > (int64_t(1) << 20) || (page_size & (page_size - 1)) != 0)
        return ATTN_ERR_INVALID_ARG;
    if (max_kv_len < Tnew || max_kv_len > max_pages * page_size || num_pages == 0)
        return ATTN_ERR_INVALID_ARG;
    if (!page_table || !kv_lens || !aligned4(page_table) || !aligned4(kv_lens))
        return ATTN_ERR_INVALID_ARG;
    const Problem pb = paged_problem(dtype, B, H, Hkv, Tnew, d, max_kv_len);
    Plan pl;
    attn_status_t st = make_plan(pb, pl);
    if (st != ATTN_OK) return st;
    if (pl.kernel != ATTN_KERNEL_SPLITKV && pl.kernel != ATTN_KERNEL_TCGEN05) return ATTN_ERR_UNSUPPORTED;
    st = check_pointers(pb, q, k_pages, v_pages, o, lse);
    if (st != ATTN_OK) return st;
    if (num_pages * Hkv * page_size * d > (int64_t(1) << 46) || num_pages * Hkv >= (int64_t(1) << 31))
        return ATTN_ERR_UNSUPPORTED;
    if (pl.ws_bytes > 0) {
        if (!workspace || workspace_bytes < pl.ws_bytes) return ATTN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
    }
    PagedKV pk;
    pk.page_table = page_table;
    pk.kv_lens = kv_lens;
    pk.max_pages = max_pages;
    pk.num_pages = num_pages;
    while ((int64_t(1) << pk.page_shift) < page_size) ++pk.page_shift;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pl.kernel == ATTN_KERNEL_TCGEN05) {
        const bool bf16 = dtype == ATTN_BF16;
        if (pl.dch == 1)
            return bf16 ? launch_prefill_paged<__nv_bfloat16, 1>(pb, pl, q, k_pages, v_pages, o, lse, scale, pk,
                                                                 page_size, workspace, s)
                        : launch_prefill_paged<__half, 1>(pb, pl, q, k_pages, v_pages, o, lse, scale, pk,
                                                          page_size, workspace, s);
        return bf16 ? launch_prefill_paged<__nv_bfloat16, 2>(pb, pl, q, k_pages, v_pages, o, lse, scale, pk,
                                                             page_size, workspace, s)
                    : launch_prefill_paged<__half, 2>(pb, pl, q, k_pages, v_pages, o, lse, scale, pk,
                                                      page_size, workspace, s);
    }
    if (dtype == ATTN_BF16)
        return run_decode<__nv_bfloat16>(pb, pl, q, k_pages, v_pages, o, lse, scale, workspace, s, &pk);
    return run_decode<__half>(pb, pl, q, k_pages, v_pages, o, lse, scale, workspace, s, &pk);
}

size_t attn_cached_paged_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                                        int64_t Tnew, int64_t d, int64_t max_kv_len) {
    if (Tnew < 0 || max_kv_len < Tnew) return 0;
    Plan pl;
    if (make_plan(paged_problem(dtype, B, H, Hkv, Tnew, d, max_kv_len), pl) != ATTN_OK) return 0;
    return pl.ws_bytes;
}

attn_status_t attn_prefill_local(const void* q, const void* k, const void* v, void* o, float* lse,
                                 attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv, int64_t T,
                                 int64_t d, float scale, int64_t window, void* stream) {
    Problem pb{dtype, B, H, Hkv, T, T, T, d, 0, 1, false, window};
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    Plan pl;
    attn_status_t st = make_plan(pb, pl);
    if (st != ATTN_OK) return st;
    st = check_pointers(pb, q, k, v, o, lse);
    if (st != ATTN_OK) return st;
    return dispatch(pb, pl, q, k, v, o, lse, scale, nullptr, static_cast<cudaStream_t>(stream));
}

attn_status_t attn_cached_local(const void* q, const void* k_hist, const void* v_hist, void* o,
                                float* lse, attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                                int64_t Tnew, int64_t S, int64_t S_cap, int64_t d,
                                int64_t start_pos, float scale, int64_t window, void* workspace,
                                size_t workspace_bytes, void* stream) {
    Problem pb{dtype, B, H, Hkv, Tnew, S, S_cap, d, start_pos, 1, true, window};
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    Plan pl;
    attn_status_t st = make_plan(pb, pl);
    if (st != ATTN_OK) return st;
    st = check_pointers(pb, q, k_hist, v_hist, o, lse);
    if (st != ATTN_OK) return st;
    if (pl.ws_bytes > 0) {
        if (!workspace || workspace_bytes < pl.ws_bytes) return ATTN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
    }
    return dispatch(pb, pl, q, k_hist, v_hist, o, lse, scale, workspace,
                    static_cast<cudaStream_t>(stream));
}

size_t attn_cached_local_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                                        int64_t Tnew, int64_t S, int64_t d, int64_t start_pos,
                                        int64_t window) {
    Problem pb{dtype, B, H, Hkv, Tnew, S, S, d, start_pos, 1, true, window};
    Plan pl;
    if (make_plan(pb, pl) != ATTN_OK) return 0;
    return pl.ws_bytes;
}

size_t attn_cached_workspace_size(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                                  int64_t Tnew, int64_t S, int64_t d, int64_t start_pos) {
    Problem pb{dtype, B, H, Hkv, Tnew, S, S, d, start_pos, 1, true};
    Plan pl;
    if (make_plan(pb, pl) != ATTN_OK) return 0;
    return pl.ws_bytes;
}

attn_kernel_t attn_prefill_plan(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv, int64_t T,
                                int64_t d, int causal) {
    Problem pb{dtype, B, H, Hkv, T, T, T, d, 0, causal ? 1 : 0, false};
    Plan pl;
    if (make_plan(pb, pl) != ATTN_OK) return static_cast<attn_kernel_t>(-1);
    return pl.kernel;
}

attn_kernel_t attn_cached_plan(attn_dtype_t dtype, int64_t B, int64_t H, int64_t Hkv,
                               int64_t Tnew, int64_t S, int64_t S_cap, int64_t d,
                               int64_t start_pos) {
    Problem pb{dtype, B, H, Hkv, Tnew, S, S_cap, d, start_pos, 1, true};
    Plan pl;
    if (make_plan(pb, pl) != ATTN_OK) return static_cast<attn_kernel_t>(-1);
    return pl.kernel;
}

const char* attn_status_string(attn_status_t status) {
    switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape";
    case ATTN_ERR_WORKSPACE: return "workspace too small";
    case ATTN_ERR_CUDA: return "CUDA runtime error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a device-side wait timed out";
    case ATTN_ERR_DEVICE_INDEX: return "a page table or length entry was out of range";
    }
    return "unknown status";
}

attn_status_t attn_device_status(void* stream, int reset) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int value = 0;
    if (cudaMemcpyFromSymbolAsync(&value, g_device_status, sizeof(value), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
    if (reset && value != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(zero), 0,
                                    cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return ATTN_ERR_CUDA;
    }
    return static_cast<attn_status_t>(value);
}

void attn_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns ? ns : kDefaultTimeoutNs); }

void attn_test_set_flags(uint32_t flags) { g_test_flags.store(flags); }

int attn_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// attn_cached_noalloc: the cached entry point for callers that may not
// allocate device memory.  Its only scratch need (the split-KV partials) is
// served from this fixed array, which lives in every device that loads the
// library until the process exits.  The decode kernel writes every partial it
// later reads, so nothing in the array has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;

// The scratch array's device address, per device, with the id of the context
// it was looked up in.
struct NoallocAddress {
    unsigned long long ctx_id = 0;
    void* ptr = nullptr;
};
NoallocAddress g_noalloc_addr[kNoAllocMaxDevices];

// Process-unique id of the current context (context ids are never reused
// while the process lives), through the driver entry points.
attn_status_t current_context_id(unsigned long long* id) {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
    });
    if (!get_current || !get_id) return ATTN_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return ATTN_ERR_CUDA;
    return get_id(ctx, id) == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// Device address of the scratch array on the current device.  The host-side
// name is only a handle for the runtime; the address is looked up with
// cudaGetSymbolAddress (with the device current) the first time a device is
// used in a context and kept for that context.  A device reset ends the
// context and reloads the module elsewhere: the next call sees a new context
// id and looks the address up again.
attn_status_t noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
        return ATTN_ERR_CUDA;
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx) == ATTN_OK;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoallocAddress& a = g_noalloc_addr[dev];
    if (!have_ctx || !a.ptr || a.ctx_id != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
        // the lookup has made the device's context current if it was not yet
        if (current_context_id(&ctx) != ATTN_OK) return ATTN_ERR_CUDA;
        a.ptr = p;
        a.ctx_id = ctx;
    }
    *out = a.ptr;
    return ATTN_OK;
}

}  // namespace

extern "C" attn_status_t attn_cached_noalloc(const void* q, const void* k_hist,
                                             const void* v_hist, void* o, float* lse,
                                             attn_dtype_t dtype, int64_t B, int64_t H,
                                             int64_t Hkv, int64_t Tnew, int64_t S, int64_t S_cap,
                                             int64_t d, int64_t start_pos, float scale,
                                             void* stream) {
    Problem pb{dtype, B, H, Hkv, Tnew, S, S_cap, d, start_pos, 1, true};
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    Plan pl;
    attn_status_t st = make_plan(pb, pl, ATTN_NOALLOC_SCRATCH_BYTES);
    if (st != ATTN_OK) return st;
    st = check_pointers(pb, q, k_hist, v_hist, o, lse);
    if (st != ATTN_OK) return st;
    if (pl.ws_bytes > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    if (pl.kernel == ATTN_KERNEL_NONE) return ATTN_OK;
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != ATTN_OK) return st;
    return dispatch(pb, pl, q, k_hist, v_hist, o, lse, scale, pl.ws_bytes ? scratch : nullptr,
                    static_cast<cudaStream_t>(stream));
}
