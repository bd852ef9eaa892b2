// attn_api.cu -- host side of the C ABI declared in include/attn.h: argument
// validation, TMA tensor-map encoding, kernel selection and launch on the
// caller's stream.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "fwd_common.cuh"
#include "fwd_kernel_pp.cuh"
#include "bwd_kernels.cuh"
#include "decode_kernel.cuh"
#include "short_kernel.cuh"
#include "quant_kernel.cuh"

using namespace attn_sm100;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;

std::atomic<int> g_last_cuda_error{0};
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<unsigned int> g_epoch{0};

// Launch id for the launch-wide abort flag; never 0 (the flag's initial value).
unsigned int next_epoch() {
    unsigned int e = g_epoch.fetch_add(1u) + 1u;
    return e == 0u ? next_epoch() : e;
}

struct DeviceState {
    bool ready = false;
    attn_status_t status = ATTN_OK;
    int sm_count = 0;
};
constexpr int kMaxDevices = 64;
DeviceState g_dev[kMaxDevices];
std::mutex g_mutex;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

attn_status_t cuda_fail(cudaError_t e) {
    g_last_cuda_error.store(static_cast<int>(e));
    return ATTN_ERR_CUDA;
}

// Persistent two-tile kernel: d=128 keeps one Q buffer (64 KB) and 5 K/V slots
// (160 KB) for deep K/V prefetch on long sequences; d=64 double-buffers Q
// (2 x 32 KB) so that the next unit's Q loads behind the current one, with
// 8 K/V slots (128 KB).
constexpr int kSlots128 = 5, kQStages128 = 1;
constexpr int kSlots64 = 8, kQStages64 = 2;
// FP8 (d = 128): 16 KB tiles, so two Q buffers and 8 K/V slots
constexpr int kSlotsF8 = 8, kQStagesF8 = 2;
// Short-key kernel: all the shared memory a CTA may have (227 KB); the K/V
// buffers take what the key count needs and the Q ring the rest.
constexpr int kShortSmemMax = 232448;
using SmemF8 = SmemPPFor<128, kSlotsF8, kQStagesF8, true>;

template <int D, int NSLOT, int QS, bool M>
cudaError_t set_pp_attrs() {
    constexpr int kSmem = SmemPPFor<D, NSLOT, QS, false>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_pp_kernel<D, NSLOT, QS, M, false, false, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_fwd_pp_kernel<D, NSLOT, QS, M, true, false, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess || M) return e;
    return cudaFuncSetAttribute(attn_fwd_pp_kernel<D, NSLOT, QS, false, false, true, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
}

template <int D>
cudaError_t set_bwd_attrs() {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<D, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SmemBwd<D>::kAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_kernel<D, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SmemBwd<D>::kAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_kernel<D, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SmemBwd<D>::kAlloc);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(attn_bwd_kernel<D, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SmemBwd<D>::kAlloc);
}

template <int D>
cudaError_t set_decode_attrs() {
    return cudaFuncSetAttribute(attn_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SmemDec<D>::kAlloc);
}

template <int D>
cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecParams& dp, unsigned grid,
                          cudaStream_t s) {
    attn_decode_kernel<D><<<grid, kDecThreads, SmemDec<D>::kAlloc, s>>>(tk, tv, dp);
    return cudaGetLastError();
}

// One-time per-device set-up: architecture check, SM count, kernel attributes,
// and the driver's tensor-map encoder.
attn_status_t device_setup(int* dev_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
    *dev_out = dev;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState& st = g_dev[dev];
    if (st.ready) return st.status;
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return cuda_fail(e);
    if (major != 10 || minor != 0) {
        st.ready = true;
        st.status = ATTN_ERR_UNSUPPORTED;
        return st.status;
    }
    if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return cuda_fail(e);
        if (q != cudaDriverEntryPointSuccess || fn == nullptr) return ATTN_ERR_UNSUPPORTED;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if ((e = set_pp_attrs<128, kSlots128, kQStages128, false>()) != cudaSuccess) return cuda_fail(e);
    if ((e = set_pp_attrs<128, kSlots128, kQStages128, true>()) != cudaSuccess) return cuda_fail(e);
    if ((e = set_pp_attrs<64, kSlots64, kQStages64, false>()) != cudaSuccess) return cuda_fail(e);
    if ((e = set_pp_attrs<64, kSlots64, kQStages64, true>()) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaFuncSetAttribute(attn_fwd_pp_kernel<128, kSlotsF8, kQStagesF8, false, false, false, true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, SmemF8::kAlloc)) != cudaSuccess)
        return cuda_fail(e);
    if ((e = set_bwd_attrs<128>()) != cudaSuccess) return cuda_fail(e);
    if ((e = set_decode_attrs<128>()) != cudaSuccess) return cuda_fail(e);
    if ((e = set_decode_attrs<64>()) != cudaSuccess) return cuda_fail(e);
    if ((e = set_bwd_attrs<64>()) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaFuncSetAttribute(attn_fwd_short_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kShortSmemMax)) != cudaSuccess)
        return cuda_fail(e);
    st.ready = true;
    st.status = ATTN_OK;
    return ATTN_OK;
}

// 3-D map over a [heads, rows, d] bf16 tensor, box = 64 columns x 128 rows x 1,
// 128-byte swizzle (the layout the UMMA shared-memory descriptors expect).
attn_status_t encode_map_uncached(CUtensorMap* map, const void* base, int d, int rows, long long heads,
                                  unsigned box_rows, bool fp8) {
    const cuuint64_t eb = fp8 ? 1u : 2u;  // bytes per element; a box row is 128 bytes either way
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * eb, static_cast<cuuint64_t>(rows) * d * eb};
    cuuint32_t box[3] = {fp8 ? 128u : 64u, box_rows, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = g_encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error.store(static_cast<int>(r));
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

// Encoded maps are kept per (device, base, shape, box): a call on the same
// buffers as an earlier one (the usual case in a serving or training loop)
// copies a 128-byte descriptor instead of asking the driver again.  A map
// holds only the address and the layout, never data, so a stale entry is
// harmless; the table is small and replaced round-robin.
struct MapKey {
    const void* base;
    long long heads;
    int dev, d, rows;
    unsigned box_rows;
    bool fp8;
    bool operator==(const MapKey& o) const {
        return base == o.base && heads == o.heads && dev == o.dev && d == o.d && rows == o.rows &&
               box_rows == o.box_rows && fp8 == o.fp8;
    }
};
constexpr int kMapCache = 64;
struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool used;
};
MapEntry g_maps[kMapCache];
int g_map_next = 0;
std::mutex g_map_mutex;

attn_status_t encode_map(CUtensorMap* map, const void* base, int d, int rows, long long heads,
                         unsigned box_rows = 128u, bool fp8 = false) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    const MapKey key{base, heads, dev, d, rows, box_rows, fp8};
    {
        std::lock_guard<std::mutex> lock(g_map_mutex);
        for (int i = 0; i < kMapCache; ++i)
            if (g_maps[i].used && g_maps[i].key == key) {
                *map = g_maps[i].map;
                return ATTN_OK;
            }
    }
    const attn_status_t st = encode_map_uncached(map, base, d, rows, heads, box_rows, fp8);
    if (st != ATTN_OK) return st;
    std::lock_guard<std::mutex> lock(g_map_mutex);
    MapEntry& e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.key = key;
    e.map = *map;
    e.used = true;
    return ATTN_OK;
}

template <int D, int NSLOT, int QS, bool M>
cudaError_t launch_pp(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                      const FwdParams& p_in, unsigned grid, cudaStream_t stream) {
    constexpr int kSmem = SmemPPFor<D, NSLOT, QS, false>::kAlloc;
    FwdParams p = p_in;
    set_fast_divs(p);
    // A last round of two-tile units that would fill at most half the CTAs runs as
    // single-tile units, two per unit (d = 64 without causal or 2-D masks: causal
    // launches pair heavy and light units instead, and a single tile under a 2-D
    // mask would still visit the key blocks of both tiles' rectangles).
    const int n_units = p.B * p.Hq * p.n_qtiles * p.n_splits;
    const int tail = static_cast<int>(n_units % static_cast<int>(grid));
    const bool split_tail = D == 64 && p.n_splits == 1 && !p.is_causal && p.unit_run == 1 && p.m2_kind == 0 &&
                            n_units > static_cast<int>(grid) && tail > 0 && 2 * tail <= static_cast<int>(grid);
    p.n_full_units = split_tail ? n_units - tail : n_units;
    p.n_units_total = split_tail ? n_units + tail : n_units;
    if (p.n_splits > 1)
        attn_fwd_pp_kernel<D, NSLOT, QS, M, true, false, false><<<grid, kPPThreads, kSmem, stream>>>(tq, tk, tv, to, p);
    else if (!M && (p.softcap_on || p.m2_kind != 0))
        attn_fwd_pp_kernel<D, NSLOT, QS, false, false, true, false><<<grid, kPPThreads, kSmem, stream>>>(tq, tk, tv, to,
                                                                                                       p);
    else
        attn_fwd_pp_kernel<D, NSLOT, QS, M, false, false, false><<<grid, kPPThreads, kSmem, stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kWsAlign = 256;
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace of a split-KV launch: partial O (fp32, [n_splits][B*Hq*Nq][d]) then
// partial LSE (fp32, [n_splits][B*Hq*Nq]), each rounded up to 256 bytes.
size_t splitkv_bytes(long long rows, int d, int n_splits) {
    return round_up(static_cast<size_t>(n_splits) * rows * d * sizeof(float), kWsAlign) +
           round_up(static_cast<size_t>(n_splits) * rows * sizeof(float), kWsAlign);
}

// Number of key ranges: the smallest-cost choice under a plain model in which a
// wave of `sms` concurrent units takes (key blocks per range + kUnitOverhead)
// block-times, and a unit count that is not a multiple of `sms` wastes the rest
// of its last wave.  `requested` > 0 is taken as an upper bound.
constexpr int kMaxSplits = 128;
constexpr int kDecRangeCost = 15;  // chunks' worth of fixed cost per decode CTA (fitted on B200)
constexpr int kUnitOverheadBlocks = 2;
int choose_splits(long long base_units, int Nk, int sms, int requested) {
    const int n_blocks = (Nk + kBN - 1) / kBN;
    if (requested > 0) return requested < n_blocks ? requested : n_blocks;
    const int hi = kMaxSplits < n_blocks ? kMaxSplits : n_blocks;
    int best = 1;
    long long best_cost = -1;
    for (int s = 1; s <= hi; ++s) {
        const int per = (n_blocks + s - 1) / s;
        const int s_eff = (n_blocks + per - 1) / per;  // ranges that hold keys
        if (s_eff != s) continue;
        const long long waves = (base_units * s + sms - 1) / sms;
        const long long cost = waves * (per + kUnitOverheadBlocks);
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = s; }
    }
    return best;
}

// Whether a split-KV call can run on the decode kernel: every query head of a
// K/V head times Nq fits its row limit, no causal or additive mask.
bool decode_shape(int Hq, int Hkv, int Nq, bool causal, bool mask) {
    return !causal && !mask && static_cast<long long>(Hq / Hkv) * Nq <= kDecMaxRows;
}

struct SplitPlan {
    bool decode;     // decode kernel (32-key chunks) instead of the tile kernel (128-key blocks)
    int n_splits;    // key ranges
    int split_keys;  // keys per range
    size_t bytes;    // workspace
};

// The plan of a split-KV call.  Decode-shaped calls (ignoring an additive mask,
// which the caller may add without re-planning) minimise a wave-count cost; the
// others use choose_splits.  A call with a mask on a decode shape runs the
// tile kernel with at most the planned number of ranges, so the workspace fits.
SplitPlan make_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, bool causal, int requested, int sms) {
    SplitPlan pl{};
    const long long rows = static_cast<long long>(B) * Hq * Nq;
    if (decode_shape(Hq, Hkv, Nq, causal, false)) {
        const int chunks = (Nk + kDecChunk - 1) / kDecChunk;
        int n;
        if (requested > 0) {
            n = requested;
        } else {
            // one CTA per SM streams about its share of HBM bandwidth, so the time is
            // (waves of CTAs over the SMs) x (chunks per range + a fixed cost of about
            // kDecRangeCost chunks for the pipeline fill and the merge); ranges keep
            // at least one chunk per consumer warp
            const long long pairs = static_cast<long long>(B) * Hkv;
            const int most = chunks / kDecWarps > 1 ? chunks / kDecWarps : 1;
            long long best_cost = -1;
            n = 1;
            for (int t = 1; t <= most && t <= kMaxSplits; ++t) {
                const int per_t = (chunks + t - 1) / t;
                if ((chunks + per_t - 1) / per_t != t) continue;
                const long long waves = (pairs * t + sms - 1) / sms;
                const long long cost = waves * (per_t + kDecRangeCost);
                if (best_cost < 0 || cost < best_cost) { best_cost = cost; n = t; }
            }
        }
        if (n > chunks) n = chunks;
        if (n < 1) n = 1;
        const int per = (chunks + n - 1) / n;
        pl.decode = true;
        pl.n_splits = (chunks + per - 1) / per;
        pl.split_keys = per * kDecChunk;
        pl.bytes = splitkv_bytes(rows, d, pl.n_splits);
        return pl;
    }
    const long long n_qtiles = (static_cast<long long>(Nq) + 2 * kBM - 1) / (2 * kBM);
    const int chosen = choose_splits(static_cast<long long>(B) * Hq * n_qtiles, Nk, sms, requested);
    const int n_blocks = (Nk + kBN - 1) / kBN;
    const int per = (n_blocks + chosen - 1) / chosen;
    pl.decode = false;
    pl.n_splits = (n_blocks + per - 1) / per;
    pl.split_keys = per * kBN;
    pl.bytes = pl.n_splits > 1 ? splitkv_bytes(rows, d, pl.n_splits) : 0;
    return pl;
}


// The short-key kernel (short_kernel.cuh): tiles of 128 query rows, K/V of a
// head resident in shared memory across its tiles.
attn_status_t launch_short(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                           int Hkv, int Nq, int Nk, float scale_log2, int is_causal, const int32_t* key_lens,
                           unsigned long long timeout_ns, unsigned int epoch, int sm_count, void* stream) {
    ShortParams sp{};
    sp.B = B; sp.Hq = Hq; sp.Hkv = Hkv; sp.Nq = Nq; sp.Nk = Nk;
    sp.n_qt = (Nq + 127) / 128;
    sp.n_pad = (Nk + 15) / 16 * 16;
    sp.kv_bytes = sp.n_pad * 128;
    sp.tiles = static_cast<long long>(B) * Hq * sp.n_qt;
    if (sp.tiles > (1LL << 30)) return ATTN_ERR_INVALID_ARG;  // tile indices stay in int range
    const SmemShort base = SmemShort::make(sp.kv_bytes, 0);
    sp.nq_stages = (kShortSmemMax - 1024 - base.bytes) / kShortTile;
    if (sp.nq_stages > kShortMaxQ) sp.nq_stages = kShortMaxQ;
    sp.scale_log2 = scale_log2;
    sp.is_causal = is_causal ? 1 : 0;
    sp.key_lens = key_lens;
    sp.lse = lse;
    sp.out = out;
    sp.timeout_ns = timeout_ns;
    sp.epoch = epoch;
    sp.fd_qt = make_fast_div(static_cast<uint32_t>(sp.n_qt));
    sp.fd_hq = make_fast_div(static_cast<uint32_t>(Hq));
    sp.fd_group = make_fast_div(static_cast<uint32_t>(Hq / Hkv));
    CUtensorMap tq, tk, tv, to;
    attn_status_t st;
    if ((st = encode_map(&tq, q, 64, Nq, static_cast<long long>(B) * Hq)) != ATTN_OK) return st;
    if ((st = encode_map(&tk, k, 64, Nk, static_cast<long long>(B) * Hkv, static_cast<unsigned>(sp.n_pad))) != ATTN_OK)
        return st;
    if ((st = encode_map(&tv, v, 64, Nk, static_cast<long long>(B) * Hkv, static_cast<unsigned>(sp.n_pad))) != ATTN_OK)
        return st;
    if ((st = encode_map(&to, out, 64, Nq, static_cast<long long>(B) * Hq)) != ATTN_OK) return st;
    const int sms = sm_count > 0 ? sm_count : 1;
    const unsigned grid = static_cast<unsigned>(sp.tiles < sms ? sp.tiles : sms);
    const int smem = SmemShort::make(sp.kv_bytes, sp.nq_stages).bytes + 1024;
    attn_fwd_short_kernel<<<grid, kShortThreads, smem, static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, to, sp);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return ATTN_OK;
}

// Host-side argument checks of the forward entry points (no CUDA call); on
// success the element strides of the additive mask are in msb, msh, msq.
attn_status_t validate_fwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                           const int32_t* key_lens, const float* additive_mask, const int64_t* mask_strides,
                           bool split_kv, int n_splits_req, const void* workspace, const attn_score_mod_t* mod,
                           long long* msb, long long* msh, long long* msq) {
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return ATTN_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (key_lens != nullptr && additive_mask != nullptr) return ATTN_ERR_INVALID_ARG;
    if (!(std::isfinite(scale)) || scale < 0.0f) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_ALIGNMENT;
    if ((lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (key_lens != nullptr && (reinterpret_cast<uintptr_t>(key_lens) & 3u)) ||
        (additive_mask != nullptr && (reinterpret_cast<uintptr_t>(additive_mask) & 3u)))
        return ATTN_ERR_ALIGNMENT;
    *msb = *msh = *msq = 0;
    if (additive_mask != nullptr) {
        if (mask_strides != nullptr) {
            *msb = mask_strides[0];
            *msh = mask_strides[1];
            *msq = mask_strides[2];
            if (*msb < 0 || *msh < 0 || *msq < 0) return ATTN_ERR_INVALID_ARG;
        } else {
            *msq = Nk;
            *msh = static_cast<long long>(Nq) * Nk;
            *msb = *msh * Hq;
        }
    }
    if (split_kv && (n_splits_req < 0 || (workspace != nullptr && reinterpret_cast<uintptr_t>(workspace) % kWsAlign)))
        return n_splits_req < 0 ? ATTN_ERR_INVALID_ARG : ATTN_ERR_ALIGNMENT;
    const bool use_mod = mod != nullptr && (mod->softcap != 0.0f || mod->mask2d_kind != ATTN_MASK2D_NONE);
    if (mod != nullptr) {
        if (!std::isfinite(mod->softcap) || mod->softcap < 0.0f) return ATTN_ERR_INVALID_ARG;
        if (mod->mask2d_kind != ATTN_MASK2D_NONE && mod->mask2d_kind != ATTN_MASK2D_NEIGHBORHOOD &&
            mod->mask2d_kind != ATTN_MASK2D_WINDOW)
            return ATTN_ERR_INVALID_ARG;
        if (mod->mask2d_kind != ATTN_MASK2D_NONE && (mod->grid_w <= 0 || mod->size <= 0 || mod->shift < 0))
            return ATTN_ERR_INVALID_ARG;
    }
    if (use_mod && (additive_mask != nullptr || split_kv)) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// Shared by attn_fwd (n_splits = 1) and attn_fwd_splitkv.
attn_status_t fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Hq, int Hkv, int Nq, int Nk, int d,
                       float scale, int is_causal,
                       const int32_t* key_lens,
                       const float* additive_mask, const int64_t* mask_strides,
                       bool split_kv, int n_splits_req, void* workspace, size_t workspace_bytes,
                       const attn_score_mod_t* mod, void* stream) {
    // ---- host-side validation (no CUDA call before this passes)
    long long msb = 0, msh = 0, msq = 0;
    attn_status_t vst = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, key_lens, additive_mask,
                                     mask_strides, split_kv, n_splits_req, workspace, mod, &msb, &msh, &msq);
    if (vst != ATTN_OK) return vst;
    const bool use_mod = mod != nullptr && (mod->softcap != 0.0f || mod->mask2d_kind != ATTN_MASK2D_NONE);

    int dev = 0;
    attn_status_t st = device_setup(&dev);
    if (st != ATTN_OK) return st;

    float scale_eff = scale == 0.0f ? static_cast<float>(1.0 / std::sqrt(static_cast<double>(d))) : scale;
    FwdParams p;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk;
    p.group = Hq / Hkv;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale_eff) * 1.4426950408889634);
    p.is_causal = is_causal ? 1 : 0;
    p.key_lens = key_lens;
    p.mask = additive_mask;
    p.msb = msb; p.msh = msh; p.msq = msq;
    p.lse = lse;
    p.out = out;
    p.unit_run = 1;
    p.softcap_on = 0;
    p.sc_in = 0.0f;
    p.sc_out = 0.0f;
    p.m2_kind = 0;
    p.m2_w = 1;
    p.m2_size = 1;
    p.m2_shift = 0;
    p.q_scale = p.k_scale = p.v_scale = nullptr;
    p.nqb = p.nkb = 0;
    if (use_mod) {
        if (mod->softcap > 0.0f) {
            // the kernel turns each raw score into the base-2 logit cap*log2(e)*tanh(scale*s/cap),
            // so the later steps use a unit scale
            p.softcap_on = 1;
            p.sc_in = static_cast<float>(2.0 * scale_eff * 1.4426950408889634 / mod->softcap);
            p.sc_out = static_cast<float>(static_cast<double>(mod->softcap) * 1.4426950408889634);
            p.sc_a = static_cast<float>(static_cast<double>(scale_eff) / mod->softcap);
            p.sc_lim = static_cast<float>(kTanhPolyRange * static_cast<double>(mod->softcap) / scale_eff);
            for (int i = 0; i < kTanhPolyTerms; ++i)
                p.sc_poly[i] = static_cast<float>(scale_eff * 1.4426950408889634 * kTanhPoly[i]);
            p.scale_log2 = 1.0f;
        }
        p.m2_kind = mod->mask2d_kind;
        if (p.m2_kind != ATTN_MASK2D_NONE) {
            p.m2_w = mod->grid_w;
            p.m2_size = mod->size;
            p.m2_shift = mod->shift;
        }
    }
    p.timeout_ns = g_timeout_ns.load();
    p.epoch = next_epoch();

    // Short key sequences (d = 64, at most 256 keys, no additive mask or variant,
    // one key range): the whole score row of a tile fits one tensor-memory
    // accumulator, so the short-key kernel runs the exact softmax without rescaling.
    if (d == 64 && Nk <= kShortMaxKeys && additive_mask == nullptr && !use_mod &&
        (!split_kv || make_plan(B, Hq, Hkv, Nq, Nk, d, is_causal != 0, n_splits_req,
                                g_dev[dev].sm_count > 0 ? g_dev[dev].sm_count : 1).n_splits == 1))
        return launch_short(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, p.scale_log2, is_causal, key_lens,
                            p.timeout_ns, p.epoch, g_dev[dev].sm_count, stream);

    CUtensorMap tq, tk, tv, to;
    if ((st = encode_map(&tq, q, d, Nq, static_cast<long long>(B) * Hq)) != ATTN_OK) return st;
    if ((st = encode_map(&tk, k, d, Nk, static_cast<long long>(B) * Hkv)) != ATTN_OK) return st;
    if ((st = encode_map(&tv, v, d, Nk, static_cast<long long>(B) * Hkv)) != ATTN_OK) return st;
    if ((st = encode_map(&to, out, d, Nq, static_cast<long long>(B) * Hq)) != ATTN_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool has_mask = additive_mask != nullptr;
    cudaError_t e;
    // Work units of 256 query rows (two tiles sharing each K/V block); one
    // persistent CTA per SM loops over them.
    p.n_qtiles = static_cast<int>((static_cast<long long>(Nq) + 2 * kBM - 1) / (2 * kBM));
    const int sms = g_dev[dev].sm_count > 0 ? g_dev[dev].sm_count : 1;
    const long long rows = static_cast<long long>(B) * Hq * Nq;
    p.n_splits = 1;
    p.split_keys = (Nk + kBN - 1) / kBN * kBN;
    p.ws_o = nullptr;
    p.ws_lse = nullptr;
    if (split_kv) {
        const SplitPlan pl = make_plan(B, Hq, Hkv, Nq, Nk, d, is_causal != 0, n_splits_req, sms);
        if (pl.decode && additive_mask == nullptr) {
            if (workspace == nullptr || workspace_bytes < pl.bytes) return ATTN_ERR_INVALID_ARG;
            DecParams dp;
            dp.B = B; dp.Hq = Hq; dp.Hkv = Hkv; dp.Nq = Nq; dp.Nk = Nk; dp.group = Hq / Hkv;
            dp.rows = dp.group * Nq;
            dp.scale_log2 = p.scale_log2;
            dp.key_lens = key_lens;
            dp.q = static_cast<const uint16_t*>(q);
            dp.n_splits = pl.n_splits;
            dp.split_keys = pl.split_keys;
            dp.ws_o = static_cast<float*>(workspace);
            dp.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                 round_up(static_cast<size_t>(pl.n_splits) * rows * d * sizeof(float),
                                                          kWsAlign));
            dp.timeout_ns = p.timeout_ns;
            dp.epoch = p.epoch;
            CUtensorMap dk, dv;
            if ((st = encode_map(&dk, k, d, Nk, static_cast<long long>(B) * Hkv, kDecChunk)) != ATTN_OK) return st;
            if ((st = encode_map(&dv, v, d, Nk, static_cast<long long>(B) * Hkv, kDecChunk)) != ATTN_OK) return st;
            cudaStream_t s = static_cast<cudaStream_t>(stream);
            const unsigned grid = static_cast<unsigned>(static_cast<long long>(B) * Hkv * pl.n_splits);
            cudaError_t e;
            e = d == 128 ? launch_decode<128>(dk, dv, dp, grid, s) : launch_decode<64>(dk, dv, dp, grid, s);
            if (e != cudaSuccess) return cuda_fail(e);
            const unsigned cg = static_cast<unsigned>((rows + 7) / 8);
            if (d == 128)
                attn_splitkv_combine_kernel<128><<<cg, 256, 0, s>>>(dp.ws_o, dp.ws_lse, static_cast<__nv_bfloat16*>(out),
                                                                    lse, rows, pl.n_splits);
            else
                attn_splitkv_combine_kernel<64><<<cg, 256, 0, s>>>(dp.ws_o, dp.ws_lse, static_cast<__nv_bfloat16*>(out),
                                                                   lse, rows, pl.n_splits);
            if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
            return ATTN_OK;
        }
        // tile kernel: at most the planned number of ranges, in 128-key blocks
        const int n_blocks = (Nk + kBN - 1) / kBN;
        const int n_splits = pl.n_splits < n_blocks ? pl.n_splits : n_blocks;
        const int per = (n_blocks + n_splits - 1) / n_splits;
        p.n_splits = (n_blocks + per - 1) / per;
        if (p.n_splits > 1) {
            p.split_keys = per * kBN;
            if (workspace == nullptr || workspace_bytes < splitkv_bytes(rows, d, p.n_splits))
                return ATTN_ERR_INVALID_ARG;
            p.ws_o = static_cast<float*>(workspace);
            p.ws_lse = reinterpret_cast<float*>(
                static_cast<char*>(workspace) +
                round_up(static_cast<size_t>(p.n_splits) * rows * d * sizeof(float), kWsAlign));
        }
    }
    const long long n_units = static_cast<long long>(B) * Hq * p.n_qtiles * p.n_splits;
    if (n_units > (1LL << 30)) return ATTN_ERR_INVALID_ARG;  // unit sequence positions stay in int range
    // Causal units differ in cost: with at least two units per SM, each CTA
    // takes heavy/light pairs of one head (equal cost per pair).
    p.unit_run = (is_causal && n_units >= 2LL * sms) ? 2 : 1;
    const long long want = (n_units + p.unit_run - 1) / p.unit_run;
    const unsigned g = static_cast<unsigned>(want < sms ? want : sms);
    if (d == 128)
        e = has_mask ? launch_pp<128, kSlots128, kQStages128, true>(tq, tk, tv, to, p, g, s)
                     : launch_pp<128, kSlots128, kQStages128, false>(tq, tk, tv, to, p, g, s);
    else
        e = has_mask ? launch_pp<64, kSlots64, kQStages64, true>(tq, tk, tv, to, p, g, s)
                     : launch_pp<64, kSlots64, kQStages64, false>(tq, tk, tv, to, p, g, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (p.n_splits > 1) {
        // merge the key ranges' partial results into out (bf16) and lse
        const unsigned cg = static_cast<unsigned>((rows + 7) / 8);
        if (d == 128)
            attn_splitkv_combine_kernel<128><<<cg, 256, 0, s>>>(p.ws_o, p.ws_lse, static_cast<__nv_bfloat16*>(out),
                                                                lse, rows, p.n_splits);
        else
            attn_splitkv_combine_kernel<64><<<cg, 256, 0, s>>>(p.ws_o, p.ws_lse, static_cast<__nv_bfloat16*>(out),
                                                               lse, rows, p.n_splits);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
    }
    return ATTN_OK;
}

// y[i] = exp2_poly_x2(x[i]), two elements per thread (the FP8 softmax's
// FMA-pipe exponential, exposed for its accuracy test).
__global__ void attn_exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    const long long i = 2LL * (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const bool two = i + 1 < n;
    const uint64_t r = exp2_poly_x2(pack_f32x2(x[i], two ? x[i + 1] : x[i]));
    y[i] = lo_f32(r);
    if (two) y[i + 1] = hi_f32(r);
}

}  // namespace

extern "C" {

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Hq, int Hkv, int Nq, int Nk, int d,
                       float scale, int is_causal,
                       const int32_t* key_lens,
                       const float* additive_mask, const int64_t* mask_strides,
                       void* stream) {
    return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens, additive_mask,
                    mask_strides, false, 1, nullptr, 0, nullptr, stream);
}

attn_status_t attn_fwd_mod(const void* q, const void* k, const void* v, void* out, float* lse,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d,
                           float scale, int is_causal,
                           const int32_t* key_lens,
                           const attn_score_mod_t* mod,
                           void* stream) {
    if (mod == nullptr) return ATTN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens, nullptr, nullptr,
                    false, 1, nullptr, 0, mod, stream);
}

attn_status_t attn_splitkv_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int is_causal, int n_splits,
                                int sm_count, int* n_splits_out, size_t* workspace_bytes) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0 || n_splits < 0 || sm_count < 0)
        return ATTN_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    int sms = sm_count;
    if (sms == 0) {
        int dev = 0;
        attn_status_t st = device_setup(&dev);
        if (st != ATTN_OK) return st;
        sms = g_dev[dev].sm_count > 0 ? g_dev[dev].sm_count : 1;
    }
    const SplitPlan pl = make_plan(B, Hq, Hkv, Nq, Nk, d, is_causal != 0, n_splits, sms);
    if (n_splits_out != nullptr) *n_splits_out = pl.n_splits;
    if (workspace_bytes != nullptr) *workspace_bytes = pl.bytes;
    return ATTN_OK;
}

attn_status_t attn_fwd_splitkv(const void* q, const void* k, const void* v, void* out, float* lse,
                               int B, int Hq, int Hkv, int Nq, int Nk, int d,
                               float scale, int is_causal,
                               const int32_t* key_lens,
                               const float* additive_mask, const int64_t* mask_strides,
                               int n_splits, void* workspace, size_t workspace_bytes,
                               void* stream) {
    return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens, additive_mask,
                    mask_strides, true, n_splits, workspace, workspace_bytes, nullptr, stream);
}

attn_status_t attn_check_device_status(void* stream, uint32_t* info) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int word = 0;
    if ((e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word))) != cudaSuccess) return cuda_fail(e);
    if (info != nullptr) *info = word;
    if (word == 0u) return ATTN_OK;
    const unsigned int zero = 0u;
    if ((e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero))) != cudaSuccess) return cuda_fail(e);
    return (word & 0xffu) == kErrTimeout ? ATTN_ERR_TIMEOUT : ATTN_ERR_DEVICE;
}

attn_status_t attn_set_wait_timeout_ns(uint64_t ns) {
    g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : static_cast<unsigned long long>(ns));
    return ATTN_OK;
}

attn_status_t attn_selftest_timeout(void* stream) {
    int dev = 0;
    attn_status_t st = device_setup(&dev);
    if (st != ATTN_OK) return st;
    attn_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(g_timeout_ns.load(), next_epoch());
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return ATTN_OK;
}

attn_status_t attn_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
    if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u)) return ATTN_ERR_ALIGNMENT;
    if (n == 0) return ATTN_OK;
    int dev = 0;
    attn_status_t st = device_setup(&dev);
    if (st != ATTN_OK) return st;
    const long long pairs = (static_cast<long long>(n) + 1) / 2;
    const unsigned grid = static_cast<unsigned>((pairs + 255) / 256);
    attn_exp2_poly_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return ATTN_OK;
}

const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported head dimension or device (needs d in {64,128} on sm_100)";
        case ATTN_ERR_ALIGNMENT: return "tensor base pointer not 16-byte aligned";
        case ATTN_ERR_CUDA: return "CUDA runtime or driver error (see attn_last_cuda_error)";
        case ATTN_ERR_TIMEOUT: return "a bounded wait inside a kernel expired";
        case ATTN_ERR_DEVICE: return "device-side consistency check failed";
        case ATTN_ERR_SCRATCH: return "the split plan needs more than the library's fixed scratch buffer "
                                      "(ATTN_NOALLOC_SCRATCH_BYTES); use attn_fwd_splitkv or fewer ranges";
        default: return "unknown status";
    }
}

int attn_last_cuda_error(void) { return g_last_cuda_error.load(); }

int attn_version(void) { return kVersion; }

}  // extern "C"

// ------------------------------------------------------------------------
// FP8 forward.
extern "C" attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
                                      const float* k_scale, const float* v_scale, void* out, float* lse,
                                      int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                      float scale, int is_causal, const int32_t* key_lens, void* stream) {
    if (q8 == nullptr || k8 == nullptr || v8 == nullptr || q_scale == nullptr || k_scale == nullptr ||
        v_scale == nullptr || out == nullptr)
        return ATTN_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (!(std::isfinite(scale)) || scale < 0.0f) return ATTN_ERR_INVALID_ARG;
    if (d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(q_scale) & 3u) || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3u) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (key_lens != nullptr && (reinterpret_cast<uintptr_t>(key_lens) & 3u)))
        return ATTN_ERR_ALIGNMENT;
    int dev = 0;
    attn_status_t st = device_setup(&dev);
    if (st != ATTN_OK) return st;
    const float scale_eff = scale == 0.0f ? static_cast<float>(1.0 / std::sqrt(static_cast<double>(d))) : scale;
    FwdParams p{};
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk;
    p.group = Hq / Hkv;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale_eff) * 1.4426950408889634);
    p.is_causal = is_causal ? 1 : 0;
    p.key_lens = key_lens;
    p.lse = lse;
    p.out = out;
    p.n_splits = 1;
    p.split_keys = (Nk + kBN - 1) / kBN * kBN;
    p.m2_w = p.m2_size = 1;
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.nqb = (Nq + kBM - 1) / kBM;
    p.nkb = (Nk + kBN - 1) / kBN;
    p.timeout_ns = g_timeout_ns.load();
    p.epoch = next_epoch();
    CUtensorMap tq, tk, tv;
    if ((st = encode_map(&tq, q8, d, Nq, static_cast<long long>(B) * Hq, 128u, true)) != ATTN_OK) return st;
    if ((st = encode_map(&tk, k8, d, Nk, static_cast<long long>(B) * Hkv, 128u, true)) != ATTN_OK) return st;
    if ((st = encode_map(&tv, v8, d, Nk, static_cast<long long>(B) * Hkv, 128u, true)) != ATTN_OK) return st;
    p.n_qtiles = static_cast<int>((static_cast<long long>(Nq) + 2 * kBM - 1) / (2 * kBM));
    const long long n_units = static_cast<long long>(B) * Hq * p.n_qtiles;
    if (n_units > (1LL << 30)) return ATTN_ERR_INVALID_ARG;
    const int sms = g_dev[dev].sm_count > 0 ? g_dev[dev].sm_count : 1;
    p.unit_run = (is_causal && n_units >= 2LL * sms) ? 2 : 1;
    const long long want = (n_units + p.unit_run - 1) / p.unit_run;
    const unsigned g = static_cast<unsigned>(want < sms ? want : sms);
    set_fast_divs(p);
    p.n_full_units = p.n_units_total = static_cast<int>(n_units);
    attn_fwd_pp_kernel<128, kSlotsF8, kQStagesF8, false, false, false, true>
        <<<g, kPPThreads, SmemF8::kAlloc, static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, tq, p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return ATTN_OK;
}

// ------------------------------------------------------------------------
// Backward pass.
namespace {

constexpr int kBwdRowPad = 128;

size_t bwd_bytes(int B, int Hq, int Nq) {
    const long long nq_pad = (static_cast<long long>(Nq) + kBwdRowPad - 1) / kBwdRowPad * kBwdRowPad;
    return 2 * round_up(static_cast<size_t>(B) * Hq * nq_pad * sizeof(float), kWsAlign);
}

template <int D, bool VAR>
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                       const BwdParams& p, cudaStream_t s) {
    const long long rows = static_cast<long long>(p.B) * p.Hq * p.nq_pad;
    attn_bwd_prep_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const dim3 g_kv((p.Nk + kBN - 1) / kBN, p.B * p.Hkv);
    attn_bwd_kernel<D, true, VAR><<<g_kv, kBwdThreads, SmemBwd<D>::kAlloc, s>>>(tq, tk, tv, tdo, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 g_q((p.Nq + kBM - 1) / kBM, p.B * p.Hq);
    attn_bwd_kernel<D, false, VAR><<<g_q, kBwdThreads, SmemBwd<D>::kAlloc, s>>>(tq, tk, tv, tdo, p);
    return cudaGetLastError();
}

}  // namespace

extern "C" attn_status_t attn_bwd_plan(int B, int Hq, int Nq, size_t* workspace_bytes) {
    if (B <= 0 || Hq <= 0 || Nq <= 0 || workspace_bytes == nullptr) return ATTN_ERR_INVALID_ARG;
    *workspace_bytes = bwd_bytes(B, Hq, Nq);
    return ATTN_OK;
}

extern "C" attn_status_t attn_bwd_ex(const void* q, const void* k, const void* v, const void* out, const float* lse,
                                     const void* dout, void* dq, void* dk, void* dv,
                                     int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                     float scale, int is_causal, const int32_t* key_lens,
                                     const float* additive_mask, const int64_t* mask_strides,
                                     const attn_score_mod_t* mod,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr || dout == nullptr ||
        dq == nullptr || dk == nullptr || dv == nullptr || workspace == nullptr)
        return ATTN_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (!(std::isfinite(scale)) || scale < 0.0f) return ATTN_ERR_INVALID_ARG;
    if (key_lens != nullptr && additive_mask != nullptr) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
        (key_lens != nullptr && (reinterpret_cast<uintptr_t>(key_lens) & 3u)) ||
        (additive_mask != nullptr && (reinterpret_cast<uintptr_t>(additive_mask) & 3u)) ||
        reinterpret_cast<uintptr_t>(workspace) % kWsAlign != 0)
        return ATTN_ERR_ALIGNMENT;
    if (workspace_bytes < bwd_bytes(B, Hq, Nq)) return ATTN_ERR_INVALID_ARG;
    long long msb = 0, msh = 0, msq = 0;
    if (additive_mask != nullptr) {
        if (mask_strides != nullptr) {
            msb = mask_strides[0];
            msh = mask_strides[1];
            msq = mask_strides[2];
            if (msb < 0 || msh < 0 || msq < 0) return ATTN_ERR_INVALID_ARG;
        } else {
            msq = Nk;
            msh = static_cast<long long>(Nq) * Nk;
            msb = msh * Hq;
        }
    }
    const bool use_mod = mod != nullptr && (mod->softcap != 0.0f || mod->mask2d_kind != ATTN_MASK2D_NONE);
    if (mod != nullptr) {
        if (!std::isfinite(mod->softcap) || mod->softcap < 0.0f) return ATTN_ERR_INVALID_ARG;
        if (mod->mask2d_kind != ATTN_MASK2D_NONE && mod->mask2d_kind != ATTN_MASK2D_NEIGHBORHOOD &&
            mod->mask2d_kind != ATTN_MASK2D_WINDOW)
            return ATTN_ERR_INVALID_ARG;
        if (mod->mask2d_kind != ATTN_MASK2D_NONE && (mod->grid_w <= 0 || mod->size <= 0 || mod->shift < 0))
            return ATTN_ERR_INVALID_ARG;
    }
    if (use_mod && additive_mask != nullptr) return ATTN_ERR_UNSUPPORTED;  // as attn_fwd_mod
    int dev = 0;
    attn_status_t st = device_setup(&dev);
    if (st != ATTN_OK) return st;

    const float scale_eff = scale == 0.0f ? static_cast<float>(1.0 / std::sqrt(static_cast<double>(d))) : scale;
    BwdParams p{};
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk; p.group = Hq / Hkv;
    p.nq_pad = (Nq + kBwdRowPad - 1) / kBwdRowPad * kBwdRowPad;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale_eff) * 1.4426950408889634);
    p.scale = scale_eff;
    p.is_causal = is_causal ? 1 : 0;
    p.key_lens = key_lens;
    p.lse = lse;
    p.o = static_cast<const uint16_t*>(out);
    p.dout = static_cast<const uint16_t*>(dout);
    p.delta = static_cast<float*>(workspace);
    p.lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + bwd_bytes(B, Hq, Nq) / 2);
    p.dq = static_cast<uint16_t*>(dq);
    p.dk = static_cast<uint16_t*>(dk);
    p.dv = static_cast<uint16_t*>(dv);
    p.timeout_ns = g_timeout_ns.load();
    p.epoch = next_epoch();
    p.mask = additive_mask;
    p.msb = msb; p.msh = msh; p.msq = msq;
    p.softcap_on = 0;
    p.m2_kind = 0;
    p.m2_w = p.m2_size = 1;
    p.m2_shift = 0;
    if (use_mod) {
        if (mod->softcap > 0.0f) {
            p.softcap_on = 1;
            p.sc_in = static_cast<float>(2.0 * scale_eff * 1.4426950408889634 / mod->softcap);
            p.sc_out = static_cast<float>(static_cast<double>(mod->softcap) * 1.4426950408889634);
        }
        if (mod->mask2d_kind != ATTN_MASK2D_NONE) {
            p.m2_kind = mod->mask2d_kind;
            p.m2_w = mod->grid_w;
            p.m2_size = mod->size;
            p.m2_shift = mod->shift;
        }
    }
    p.fd_w = make_fast_div(static_cast<uint32_t>(p.m2_w));
    p.fd_size = make_fast_div(static_cast<uint32_t>(p.m2_size));
    const bool var = use_mod || additive_mask != nullptr;

    CUtensorMap tq, tk, tv, tdo;
    if ((st = encode_map(&tq, q, d, Nq, static_cast<long long>(B) * Hq)) != ATTN_OK) return st;
    if ((st = encode_map(&tk, k, d, Nk, static_cast<long long>(B) * Hkv)) != ATTN_OK) return st;
    if ((st = encode_map(&tv, v, d, Nk, static_cast<long long>(B) * Hkv)) != ATTN_OK) return st;
    if ((st = encode_map(&tdo, dout, d, Nq, static_cast<long long>(B) * Hq)) != ATTN_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (d == 128)
        e = var ? launch_bwd<128, true>(tq, tk, tv, tdo, p, s) : launch_bwd<128, false>(tq, tk, tv, tdo, p, s);
    else
        e = var ? launch_bwd<64, true>(tq, tk, tv, tdo, p, s) : launch_bwd<64, false>(tq, tk, tv, tdo, p, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return ATTN_OK;
}

extern "C" attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                                  const void* dout, void* dq, void* dk, void* dv,
                                  int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                  float scale, int is_causal, const int32_t* key_lens,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    return attn_bwd_ex(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens,
                       nullptr, nullptr, nullptr, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------------
// Split-KV without caller memory: the workspace lives in a fixed device array
// of this library (allocated with the module, never by a call).  Serves
// callers that cannot provide device memory per call: C hosts that own no
// device allocator, servers whose memory is fully reserved up front, and
// decode loops that must not call cudaMalloc / cudaFree (which may
// synchronise the device).  Calls overlapping on one device share the array
// and race.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch for the current device, looked up once
// per device (with that device current).
attn_status_t noalloc_scratch(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        if (ptr == nullptr || reinterpret_cast<uintptr_t>(ptr) % kWsAlign != 0) return ATTN_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return ATTN_OK;
}

}  // namespace

extern "C" attn_status_t attn_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* out,
                                                  float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                                  float scale, int is_causal, const int32_t* key_lens,
                                                  const float* additive_mask, const int64_t* mask_strides,
                                                  int n_splits, void* stream) {
    // every argument check runs before the one-time device set-up
    long long msb = 0, msh = 0, msq = 0;
    attn_status_t st = validate_fwd(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, key_lens, additive_mask,
                                    mask_strides, true, n_splits, nullptr, nullptr, &msb, &msh, &msq);
    if (st != ATTN_OK) return st;
    int dev = 0;
    st = device_setup(&dev);
    if (st != ATTN_OK) return st;
    int used = 1;
    size_t need = 0;
    if ((st = attn_splitkv_plan(B, Hq, Hkv, Nq, Nk, d, is_causal, n_splits,
                                g_dev[dev].sm_count > 0 ? g_dev[dev].sm_count : 1, &used, &need)) != ATTN_OK)
        return st;
    if (need > static_cast<size_t>(ATTN_NOALLOC_SCRATCH_BYTES)) return ATTN_ERR_SCRATCH;
    void* scratch = nullptr;
    if ((st = noalloc_scratch(dev, &scratch)) != ATTN_OK) return st;
    // the plan above is the one fwd_impl makes for the same sizes and n_splits
    return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens, additive_mask,
                    mask_strides, true, n_splits, scratch, static_cast<size_t>(ATTN_NOALLOC_SCRATCH_BYTES), nullptr,
                    stream);
}

// ------------------------------------------------------------------------
// FP8 block quantisation (the inputs of attn_fwd_fp8 from bf16 tensors).
extern "C" attn_status_t attn_quantize_e4m3_blocks(const void* x, void* codes, float* scales, int heads, int N, int d,
                                                   void* stream) {
    if (x == nullptr || codes == nullptr || scales == nullptr || heads <= 0 || N <= 0 || d <= 0)
        return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return ATTN_ERR_ALIGNMENT;
    const long long nb = (static_cast<long long>(N) + kQuantRows - 1) / kQuantRows;
    if (nb * heads > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    int dev = 0;
    attn_status_t st = device_setup(&dev);
    if (st != ATTN_OK) return st;
    const unsigned grid = static_cast<unsigned>(nb * heads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 128)
        attn_quantize_e4m3_kernel<128><<<grid, kQuantThreads, 0, s>>>(static_cast<const uint16_t*>(x),
                                                                      static_cast<uint8_t*>(codes), scales, N,
                                                                      static_cast<int>(nb));
    else
        attn_quantize_e4m3_kernel<64><<<grid, kQuantThreads, 0, s>>>(static_cast<const uint16_t*>(x),
                                                                     static_cast<uint8_t*>(codes), scales, N,
                                                                     static_cast<int>(nb));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return ATTN_OK;
}
