// fwd_common.cuh -- definitions shared by the attention kernels and the host
// side: tile constants, launch parameters, error roles, and the self-test
// kernel whose bounded wait must expire.
#pragma once

#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int kBM = 128;          // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;          // keys per block
constexpr int kTmemCols = 512;
constexpr float kLazyTau = 8.0f;  // rescale only when the max grows by > 2^8

// tanh(t) = t * P(t^2) for |t| <= kTanhPolyRange: P of degree 5 in t^2, fitted by
// weighted least squares on 4000 Chebyshev nodes of [0, kTanhPolyRange^2], the
// weights driven towards least maximum relative error (2.9e-8 for the fit; 1.6e-7
// with float32 coefficients and Horner evaluation, against tanh in fp64).  The
// soft-capped score cap * tanh(scale * x / cap) then costs FMA-pipe work only.
constexpr int kTanhPolyTerms = 6;
constexpr float kTanhPolyRange = 0.75f;
constexpr float kTanhPoly[kTanhPolyTerms] = {1.000000000e+00f, -3.333295882e-01f, 1.332540661e-01f,
                                             -5.334442854e-02f, 1.958290674e-02f, -4.716256633e-03f};
// FP8 probabilities: a tighter threshold (stale-max factor at most 2^2) frees six
// binades of the E4M3 range, used to store P * 2^6; the largest stored value is
// then 2^8 <= 448 and normal E4M3 values reach down to 2^-12 of the row max.
constexpr float kLazyTauF8 = 2.0f;
constexpr float kPShiftF8 = 6.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Roles for error reporting.
enum : unsigned int { kRoleSoftmax = 1, kRoleProducer = 2, kRoleMma = 3, kRoleSelftest = 9 };

// Division by an invariant d >= 1 without a divide instruction ("Division by
// Invariant Integers using Multiplication", Granlund and Montgomery, PLDI 1994,
// Theorem 4.2 with N = 31): with l = ceil(log2 d) and m = floor(2^(31+l) / d) + 1,
// floor(n / d) = floor(m n / 2^(31+l)) for every 0 <= n < 2^31, and m < 2^32.
// (32-bit integer division by a run-time value goes through a reciprocal on the
// special-function unit, which the softmax keeps saturated: at each unit boundary
// a handful of them cost ~1000 cycles, measured with an instrumented copy.)
struct FastDiv {
    uint32_t m, l;
};

inline FastDiv make_fast_div(uint32_t d) {
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    return FastDiv{static_cast<uint32_t>((1ull << (31 + l)) / d + 1ull), l};
}

__device__ __forceinline__ int fdiv(int n, FastDiv f) {
    return static_cast<int>((static_cast<uint64_t>(f.m) * static_cast<uint32_t>(n)) >> (31 + f.l));
}

struct FwdParams {
    int B, Hq, Hkv, Nq, Nk;
    int group;          // Hq / Hkv
    int n_qtiles;       // 256-row work units per (batch, head): ceil(Nq / 256)
    float scale_log2;   // softmax scale * log2(e), > 0
    int is_causal;
    const int32_t* key_lens;
    const float* mask;
    long long msb, msh, msq;
    float* lse;
    void* out;     // O base (bf16), for rows written without the TMA store
    int unit_run;  // persistent kernel: consecutive units per CTA turn (1 or 2)
    // Units [0, n_full_units) hold two 128-row tiles; the units after them, up to
    // n_units_total, are the single tiles of the remaining two-tile units (a last
    // round that would leave SMs idle is run as twice as many half-size units).
    int n_full_units, n_units_total;
    // split-KV mode: every unit covers one range of split_keys keys (a multiple of
    // 128); partial results go to the workspace, [n_splits][B*Hq][Nq][d] for O
    // (fp32, normalised by the partial row sum) and [n_splits][B*Hq][Nq] for LSE
    int n_splits;
    int split_keys;
    float* ws_o;
    float* ws_lse;
    // score and mask variants (the MOD instantiation): soft-capped scores
    // cap * tanh(x / cap) of the scaled score x, and 2-D masks on a row-major
    // token grid of m2_w tokens per row (kind 1: neighbourhood of radius
    // m2_size, kind 2: m2_size x m2_size windows displaced by m2_shift)
    int softcap_on;
    float sc_in;   // 2 * scale * log2(e) / cap: base-2 exponent of e^(2x / cap) per raw score
    float sc_out;  // cap * log2(e)
    float sc_a;    // scale / cap: the argument of tanh per raw score
    float sc_lim;  // kTanhPolyRange / sc_a: raw scores up to this magnitude take the polynomial
    float sc_poly[kTanhPolyTerms];  // scale * log2(e) * the polynomial's coefficients
    int m2_kind, m2_w, m2_size, m2_shift;
    // FP8 instantiation: per-128-row block scales of Q [B*Hq][nqb] and K, V [B*Hkv][nkb]
    const float* q_scale;
    const float* k_scale;
    const float* v_scale;
    int nqb, nkb;
    unsigned long long timeout_ns;
    unsigned int epoch;  // launch id for the launch-wide abort (never 0)
    // divisors of the unit decode and of the 2-D masks (set by set_fast_divs)
    FastDiv fd_qtiles, fd_per_head, fd_hq, fd_group, fd_w, fd_size;
};

// Fills the FastDiv fields from the fields they divide by (host, before a launch).
inline void set_fast_divs(FwdParams& p) {
    p.fd_qtiles = make_fast_div(static_cast<uint32_t>(p.n_qtiles));
    p.fd_per_head = make_fast_div(static_cast<uint32_t>(p.n_qtiles * p.n_splits));
    p.fd_hq = make_fast_div(static_cast<uint32_t>(p.Hq));
    p.fd_group = make_fast_div(static_cast<uint32_t>(p.group));
    p.fd_w = make_fast_div(static_cast<uint32_t>(p.m2_w > 0 ? p.m2_w : 1));
    p.fd_size = make_fast_div(static_cast<uint32_t>(p.m2_size > 0 ? p.m2_size : 1));
}

// Rectangle of the token grid that query row i may see under a 2-D mask: key
// rows [r_lo, r_hi] and, within each, columns [c_lo, c_hi] (clipped to the grid).
struct Rect2D {
    int r_lo, r_hi, c_lo, c_hi;
};

__device__ __forceinline__ Rect2D rect_2d(const FwdParams& p, int i) {
    const long long W = p.m2_w;
    const long long qr = fdiv(i, p.fd_w), qc = i - qr * W;
    long long r_lo, r_hi, c_lo, c_hi;
    if (p.m2_kind == 1) {  // |dr| < R and |dc| < R
        r_lo = qr - p.m2_size + 1;
        r_hi = qr + p.m2_size - 1;
        c_lo = qc - p.m2_size + 1;
        c_hi = qc + p.m2_size - 1;
    } else {  // same displaced window
        const long long w = p.m2_size, sh = p.m2_shift;
        r_lo = static_cast<long long>(fdiv(static_cast<int>(qr + sh), p.fd_size)) * w - sh;
        r_hi = r_lo + w - 1;
        c_lo = static_cast<long long>(fdiv(static_cast<int>(qc + sh), p.fd_size)) * w - sh;
        c_hi = c_lo + w - 1;
    }
    const long long last_row = fdiv(p.Nk - 1, p.fd_w);  // key rows that exist
    Rect2D r;
    r.r_lo = static_cast<int>(r_lo < 0 ? 0 : r_lo);
    r.r_hi = static_cast<int>(r_hi > last_row ? last_row : r_hi);
    r.c_lo = static_cast<int>(c_lo < 0 ? 0 : c_lo);
    r.c_hi = static_cast<int>(c_hi > W - 1 ? W - 1 : c_hi);
    return r;
}

// Split-KV combine: for each output row, merge the n_splits partial results
// (O_s normalised by its own row sum, LSE_s) of disjoint key ranges:
//   M = max_s LSE_s,  w_s = exp(LSE_s - M),  O = sum_s w_s O_s / sum_s w_s,
//   LSE = M + ln sum_s w_s
// (exact: each w_s is proportional to the sum of exp(score) over range s).  A row
// with no key in any range gives O = 0, LSE = -inf.  One warp per row; lane i
// holds columns 4i .. 4i+3 (d = 128) or 2i .. 2i+1 (d = 64).
template <int D>
__global__ void __launch_bounds__(256) attn_splitkv_combine_kernel(const float* __restrict__ ws_o,
                                                                  const float* __restrict__ ws_lse,
                                                                  __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse, long long rows,
                                                                  int n_splits) {
    constexpr int kPer = D / 32;
    const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    float m = -INFINITY;
    for (int s = lane; s < n_splits; s += 32) m = fmaxf(m, ws_lse[s * rows + r]);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float acc[kPer];
    #pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
    float wsum = 0.0f;
    if (m != -INFINITY) {
        for (int s = 0; s < n_splits; ++s) {
            const float ls = ws_lse[s * rows + r];
            if (ls == -INFINITY) continue;
            const float w = __expf(ls - m);
            wsum += w;
            const float* src = ws_o + (s * rows + r) * D + lane * kPer;
            #pragma unroll
            for (int i = 0; i < kPer; ++i) acc[i] = fmaf(w, src[i], acc[i]);
        }
    }
    const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
    __nv_bfloat16* dst = out + r * D + lane * kPer;
    #pragma unroll
    for (int i = 0; i < kPer; i += 2)
        *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
    if (lane == 0 && lse != nullptr) lse[r] = wsum > 0.0f ? m + __logf(wsum) : -INFINITY;
}

// Waits on a barrier nothing arrives at; the bounded wait must expire.
__global__ void attn_selftest_timeout_kernel(unsigned long long timeout_ns, unsigned int epoch) {
    __shared__ __align__(8) uint64_t bar_storage;
    __shared__ int abort_storage;
    const uint32_t b = smem_u32(&bar_storage);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        abort_storage = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        mbar_wait(b, 0, timeout_ns, reinterpret_cast<volatile int*>(&abort_storage), epoch, kRoleSelftest, 1);
    __syncthreads();
}

}  // namespace attn_sm100
