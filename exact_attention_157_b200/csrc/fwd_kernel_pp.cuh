// fwd_kernel_pp.cuh -- exact attention forward pass for sm_100a: persistent
// CTAs, two query tiles per work unit ("ping-pong").
//
// Work unit = 256 query rows of one (batch, query head): tile A = rows
// q0..q0+127, tile B = rows q0+128..q0+255.  Both tiles share every K/V block,
// so K/V are read from shared memory once per 256 rows.  One CTA per SM loops
// over units.  Units are numbered head-major (the units of one head run at
// about the same time, so its K/V stay in L2); within a head, causal units
// alternate heavy and light (query tiles n-1, 0, n-2, 1, ...), and, when there
// are at least two units per CTA, every CTA takes consecutive pairs (CTA c:
// sequence positions 2(c + kG), 2(c + kG) + 1), so each CTA's causal work is a
// sum of equal-cost pairs; otherwise CTA c takes c, c + G, ...  Set-up (barriers,
// TMEM) is paid once per CTA, and the loads and MMAs of the next unit overlap
// the epilogue of the current one.
//
//   warps 0-3   softmax + epilogue of tile A (thread = row = TMEM lane)
//   warps 4-7   softmax + epilogue of tile B
//   warp 8      TMA producer: Q_A, Q_B of each unit into one of QS Q buffers,
//               K_0, V_0, K_1, V_1, ... of every unit into one ring of NSLOT
//               slots (128-byte swizzle, no multicast), in consumption order
//   warp 9      TMEM owner and MMA issuer (warp-uniform; one elected lane issues
//               each batch of MMAs and commits)
//   warp 10     aliased form: idle; decoupled form: MMA issuer of tile B
//   warp 11     idle (completes the third warpgroup that setmaxnreg needs)
//
// TMEM: S_A cols [0,128), S_B [128,256), O_A [256,256+D), O_B [256+D,256+2D).
//
// Aliased form (bf16, d = 128: tensor memory is full).  P_t (bf16 pairs, 64
// cols) overwrites the first half of S_t once the softmax has read S_t, so
// S_t(j+1) is issued after PV_t(j) by the same thread (tcgen05.mma operations
// of one thread execute in issue order):
//     S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) ...
// While the softmax of one tile runs, the tensor cores work on the other.
// Because S_t(j) is issued after PV_t(j-1), S_t(j) complete implies
// O_t = sum_{i<j} P_i V_i, so the softmax may rescale O_t right away.
//
// Decoupled form (FP8, and bf16 with d = 64).  P_t has a buffer of its own:
// FP8 in shared memory (128 rows x 128 one-byte keys, read by an SS-form MMA),
// bf16 d = 64 in the spare TMEM columns [384 + 64 t, 448 + 64 t).  The softmax
// arrives on SFREE_t as soon as S_t(j) is in registers, and the MMA warp of the
// tile issues S_t(j+1) at once, so it runs during softmax_t(j); PV_t(j) follows
// as P_t(j) is stored.  Before it stores P_t(j) or rescales O_t, the softmax
// waits for PVDONE_t (PV_t(j-1) complete).  Each K/V slot is released by both
// MMA warps (the EMPTY barriers count two); a tile past its last key block
// releases a load only once it has landed, so that the arrival cannot count
// towards the slot's previous use.
//
// Across units, PV_t(0) of the next unit waits until the epilogue has read O_t
// out of TMEM (OEMPTY), and the epilogue stages O_t through the unit's own
// (dead) Q_t buffer, which the producer refills only after the TMA store has
// read it (QEMPTY).  (FP8 writes its bf16 rows directly.)
//
// Online softmax in base 2 with the scale folded into the FMA and lazy
// rescaling ("FlashAttention technical analysis", jsqmd.com/news/722897,
// sections 2.2 and 4.1); one final normalisation; LSE = (m + log2 l) ln 2.
#pragma once

#include <type_traits>

#include "fwd_common.cuh"

namespace attn_sm100 {

constexpr int kPPThreads = 384;  // 12 warps = 3 warpgroups
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512);
// the TMA/MMA warpgroup gives back to kRegsControl and the two softmax
// warpgroups take kRegsSoftmax: 2 x 128 x 200 + 128 x 104 = 64512, exactly the
// launch total.
constexpr int kRegsSoftmax = 200;
constexpr int kRegsControl = 104;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kPPThreads * 168, "register split");

// EB: bytes per Q/K/V element (2: bf16, 1: FP8); PSMEM: P of both tiles in shared memory;
// OSTAGE: a staging buffer for the bf16 O tiles of its own (else O is staged in the dead Q buffer)
template <int D, int NSLOT, int QS, int EB = 2, bool PSMEM = false, bool OSTAGE = false>
struct SmemPP {
    static constexpr int kChunks = D * EB / 128;              // 128-byte column chunks of a row
    static constexpr int kChunkBytes = 128 * 128;
    static constexpr int kTileBytes = kChunks * kChunkBytes;  // 128 rows x D elements
    static constexpr int kQBuf = 2 * kTileBytes;              // Q_A then Q_B of one unit
    static constexpr int kQ = 0;                              // QS buffers
    static constexpr int kRing = QS * kQBuf;
    static constexpr int kPS = kRing + NSLOT * kTileBytes;   // P_A, P_B: 128 rows x 128 one-byte keys
    static constexpr int kPBytes = 128 * 128;
    static constexpr int kOS = kPS + (PSMEM ? 2 * kPBytes : 0);  // O_A, O_B staging (OSTAGE)
    static constexpr int kBars = kOS + (OSTAGE ? 2 * kTileBytes : 0);
    // barrier indices
    static constexpr int QFULL = 0;                   // QS: Q buffer loaded
    static constexpr int QEMPTY = QS;                 // QS: Q buffer free (2 arrivals: both tiles' stores)
    static constexpr int FULL = 2 * QS;               // NSLOT: K/V slot loaded
    static constexpr int EMPTY = 2 * QS + NSLOT;      // NSLOT: K/V slot released
    static constexpr int SFULL = 2 * QS + 2 * NSLOT;  // 2: S_t(j) complete
    static constexpr int P0 = SFULL + 2;              // 2: P_t(j) keys 0..63 stored (128 arrivals)
    static constexpr int P1 = SFULL + 4;              // 2: P_t(j) keys 64..127 stored (128 arrivals)
    static constexpr int OFINAL = SFULL + 6;          // 2: last PV_t of a unit complete
    static constexpr int OEMPTY = SFULL + 8;          // 2: O_t read out by the epilogue (128 arrivals)
    static constexpr int MMAFIN = SFULL + 10;
    static constexpr int SFREE = SFULL + 11;          // 2: S_t(j) read into registers (128 arrivals)
    static constexpr int PVDONE = SFULL + 13;         // 2: PV_t(j) complete (P_t buffer and O_t free)
    static constexpr int kNumBars = PVDONE + 2;
    static constexpr int kMisc = kBars + 8 * kNumBars;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kColO = 256;
    static constexpr int kColP = kColO + 2 * D;  // d = 64: P_A, P_B (64 columns each) after O
    static_assert(kColO + 2 * D <= kTmemCols, "TMEM budget");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

// The layout of one kernel instantiation; the host sizes the launch with the same alias.
template <int D, int NSLOT, int QS, bool FP8>
using SmemPPFor = SmemPP<D, NSLOT, QS, FP8 ? 1 : 2, FP8, !FP8 && D == 64>;

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}

// (a.lo*b.lo + c.lo, a.hi*b.hi + c.hi) in one instruction
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ float lo_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

// FP8 path: one pair of exponentials in every ATTN_F8_EXP_EMU is taken on the FMA
// pipe instead of the special-function unit (0: none).  With FP8 products the
// softmax warps, not the tensor cores, set the pace; one pair in four measured
// best (one in two or three was slower: the extra FMA-pipe instructions then
// cost more issue slots than the special-function unit frees).
#ifndef ATTN_F8_EXP_EMU
#define ATTN_F8_EXP_EMU 4
#endif

// 2^x for two fp32 values with FMA-pipe arithmetic only: x = n + f, n the nearest
// integer (added to the exponent field) and 2^f for |f| <= 1/2 from a cubic whose
// coefficients were fitted by the Remez exchange for least maximum relative error
// (7.5e-5 on the interval).  x < -125 (a masked key's -inf among them) gives 0, as
// ex2.approx does far below the normal range; the arithmetic itself runs on x
// clamped at -125 so that the result stays normal.
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t xv) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound holds round(x) in its low bits
    const float x0 = fmaxf(lo_f32(xv), -125.0f), x1 = fmaxf(hi_f32(xv), -125.0f);
    const uint64_t x = pack_f32x2(x0, x1);
    const uint64_t t = fadd2(x, pack_f32x2(kRound, kRound));
    const uint64_t n = fadd2(t, pack_f32x2(-kRound, -kRound));
    const uint64_t f = ffma2(n, pack_f32x2(-1.0f, -1.0f), x);
    uint64_t q = ffma2(f, pack_f32x2(0.0551716685295105f, 0.0551716685295105f),
                       pack_f32x2(0.2426111251115799f, 0.2426111251115799f));
    q = ffma2(q, f, pack_f32x2(0.6932609677314758f, 0.6932609677314758f));
    q = ffma2(q, f, pack_f32x2(0.9999280571937561f, 0.9999280571937561f));
    uint32_t r0 = static_cast<uint32_t>(q) + (static_cast<uint32_t>(t) << 23);
    uint32_t r1 = static_cast<uint32_t>(q >> 32) + (static_cast<uint32_t>(t >> 32) << 23);
    r0 = lo_f32(xv) < -125.0f ? 0u : r0;
    r1 = hi_f32(xv) < -125.0f ? 0u : r1;
    return (static_cast<uint64_t>(r1) << 32) | r0;
}

// Everything about one work unit that every role derives identically.
struct Unit {
    int bh, b, h, bhk, q0, kv_len;
    int split, j_lo;  // split-KV: key range index and its first key block
    int n_t[2];  // key blocks of tile A / B (0: nothing to compute)
    bool tile_b_valid;
    __device__ __forceinline__ int n_max() const { return n_t[0] > n_t[1] ? n_t[0] : n_t[1]; }
};

// Sequence position of the k-th unit of CTA c among G CTAs: runs of P
// consecutive units (P = 2 pairs heavy with light causal units, P = 1 is plain
// round-robin).
__device__ __forceinline__ int unit_seq(int c, int k, int G, int P) {
    return P == 2 ? 2 * (c + (k >> 1) * G) + (k & 1) : c + k * G;
}

// The key length of the batch entry of the unit at sequence position s (a
// global load, issued one unit ahead by every role so that its latency is off
// the critical path).
// FAST: the unit decode divides by multiplication (FastDiv).  Measured on B200: it
// pays where units are short and many per CTA (d = 64: vit -4 %, unet_cross -8 %
// time), and costs 2-3 % at d = 128, whose units run 32 key blocks each.
// The two-tile unit that sequence position s belongs to (s itself below
// n_full_units; a single tile of unit n_full_units + (s - n_full_units) / 2 after).
// Single-tile units exist only in the d = 64 instantiations (SINGLE); at d = 128 a
// unit runs 32 key blocks per tile and a last round costs little.
template <bool SINGLE>
__device__ __forceinline__ int unit_base(const FwdParams& p, int s) {
    if constexpr (!SINGLE) return s;
    return s < p.n_full_units ? s : p.n_full_units + ((s - p.n_full_units) >> 1);
}

template <bool FAST>
__device__ __forceinline__ int unit_key_len(const FwdParams& p, int s, int n_units) {
    if (p.key_lens == nullptr || s >= n_units) return p.Nk;
    s = unit_base<FAST>(p, s);
    if constexpr (FAST) return __ldg(p.key_lens + fdiv(fdiv(s, p.fd_per_head), p.fd_hq));
    return __ldg(p.key_lens + (s / (p.n_qtiles * p.n_splits)) / p.Hq);
}

// Units are numbered (head, split, query-unit): the units of one head and key
// range are adjacent.  Without split-KV (SPLIT = false) there is one range.
template <bool SPLIT, bool MOD, bool FAST>
__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int s, int kv_len, bool report) {
    Unit x;
    int pos;
    // a single-tile unit: 1 = the first 128 rows of its unit, 2 = the second
    const int single = !FAST || s < p.n_full_units ? 0 : 1 + ((s - p.n_full_units) & 1);
    s = unit_base<FAST>(p, s);
    if constexpr (SPLIT) {
        const int per_head = p.n_qtiles * p.n_splits;
        x.bh = FAST ? fdiv(s, p.fd_per_head) : s / per_head;
        const int r = s - x.bh * per_head;
        x.split = FAST ? fdiv(r, p.fd_qtiles) : r / p.n_qtiles;
        pos = r - x.split * p.n_qtiles;
    } else {
        x.bh = FAST ? fdiv(s, p.fd_qtiles) : s / p.n_qtiles;
        x.split = 0;
        pos = s - x.bh * p.n_qtiles;
    }
    // causal: heavy and light query tiles alternate (n-1, 0, n-2, 1, ...)
    const int qt = !p.is_causal ? pos : (pos & 1) ? (pos >> 1) : p.n_qtiles - 1 - (pos >> 1);
    x.b = FAST ? fdiv(x.bh, p.fd_hq) : x.bh / p.Hq;
    x.h = x.bh - x.b * p.Hq;
    x.bhk = x.b * p.Hkv + (FAST ? fdiv(x.h, p.fd_group) : x.h / p.group);
    x.q0 = qt * 2 * kBM;
    x.tile_b_valid = x.q0 + kBM < p.Nq;
    if (kv_len < 0 || kv_len > p.Nk) {
        if (report) record_error(kErrDevice, kRoleSoftmax, 1);
        kv_len = kv_len < 0 ? 0 : p.Nk;
    }
    x.kv_len = kv_len;
    int k_lo = SPLIT ? x.split * p.split_keys : 0;  // a multiple of kBN
    int k_hi = x.kv_len;
    if constexpr (MOD) {
        if (p.m2_kind != 0) {
            // keys of the grid rows that the unit's first and last query rows may see
            const int q_last = (x.q0 + 2 * kBM - 1 < p.Nq - 1) ? x.q0 + 2 * kBM - 1 : p.Nq - 1;
            const Rect2D a = rect_2d(p, x.q0), z = rect_2d(p, q_last);
            k_lo = (a.r_lo * p.m2_w) / kBN * kBN;
            const long long hi = (static_cast<long long>(z.r_hi) + 1) * p.m2_w;
            if (hi < k_hi) k_hi = static_cast<int>(hi);
        }
    }
    x.j_lo = k_lo / kBN;
    #pragma unroll
    for (int t = 0; t < 2; ++t) {
        int end = k_hi;
        if (p.is_causal && x.q0 + (t + 1) * kBM < end) end = x.q0 + (t + 1) * kBM;
        if (SPLIT && k_lo + p.split_keys < end) end = k_lo + p.split_keys;
        x.n_t[t] = end > k_lo ? (end - k_lo + kBN - 1) / kBN : 0;
    }
    if (!x.tile_b_valid) x.n_t[1] = 0;
    if (single != 0) {
        // (only without causal masks: both tiles of the unit see the same key blocks,
        // so tile B's count serves the single tile)
        if (single == 2) {
            x.q0 += kBM;
            x.n_t[0] = x.tile_b_valid ? x.n_t[1] : 0;
        }
        x.tile_b_valid = false;
        x.n_t[1] = 0;
    }
    return x;
}

template <int D, int NSLOT, int QS, bool HAS_MASK, bool SPLIT, bool MOD, bool FP8>
__global__ void __launch_bounds__(kPPThreads, 1)
attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdParams p) {
    using L = SmemPPFor<D, NSLOT, QS, FP8>;
    constexpr int kElemsPerChunk = FP8 ? 128 : 64;  // TMA box columns
    // Decoupled S and P: where P_t has a buffer of its own (FP8: shared memory; d = 64:
    // spare tensor-memory columns), S_t(j+1) is issued as soon as the softmax has read
    // S_t(j) into registers, so that it runs during softmax_t(j).  Otherwise (bf16,
    // d = 128, tensor memory full) P_t(j) overwrites S_t(j) and S_t(j+1) waits for PV_t(j).
    // (The additive-mask variant keeps the aliased form: it would spill registers.)
    constexpr bool kDec = FP8 || (D == 64 && !HAS_MASK);
    static_assert(!kDec || FP8 || L::kColP + 2 * 64 <= kTmemCols, "P columns");
    // A launch whose dynamic shared memory does not hold this layout touches nothing.
    uint32_t dyn_smem;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
    if (dyn_smem < static_cast<uint32_t>(L::kAlloc)) {
        if (threadIdx.x == 0) record_error(kErrDevice, kRoleSoftmax, 34);
        return;
    }
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t sbase = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // p.n_qtiles counts 256-row units per head; p.n_splits key ranges per head
    const int n_units = p.n_units_total;

    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    if (threadIdx.x == 0) {
        for (int q = 0; q < QS; ++q) {
            mbar_init(bar(L::QFULL + q), 1);
            mbar_init(bar(L::QEMPTY + q), 2);
        }
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(bar(L::FULL + s), 1);
            mbar_init(bar(L::EMPTY + s), kDec ? 2 : 1);  // decoupled: one MMA warp per tile releases
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(L::SFULL + t), 1);
            mbar_init(bar(L::P0 + t), 128);
            mbar_init(bar(L::P1 + t), 128);
            mbar_init(bar(L::OFINAL + t), 1);
            mbar_init(bar(L::OEMPTY + t), 128);
            mbar_init(bar(L::SFREE + t), 128);
            mbar_init(bar(L::PVDONE + t), 1);
        }
        mbar_init(bar(L::MMAFIN), kDec ? 2 : 1);
        *abort_flag = launch_aborted(p.epoch) ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t limit = p.timeout_ns;
    // A CTA that starts after another CTA of this launch timed out does no work.
    const int cta = __shfl_sync(0xffffffffu, *abort_flag ? n_units : static_cast<int>(blockIdx.x), 0);
    const int G = static_cast<int>(gridDim.x);

    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(kRegsControl));
      if (warp == 11 || (warp == 10 && !kDec)) {
        // idle warps
      } else if (warp == 8) {
        // ============================== TMA producer ==============================
        if (lane == 0) {
            int uses[NSLOT];
            #pragma unroll
            for (int s = 0; s < NSLOT; ++s) uses[s] = 0;
            int q_loads[QS];
            #pragma unroll
            for (int q = 0; q < QS; ++q) q_loads[q] = 0;
            int i_glob = 0;  // K/V loads issued so far (ring position)
            bool ok = true;
            int it = 0;
            int kv_next = unit_key_len<D == 64>(p, unit_seq(cta, 0, G, p.unit_run), n_units);
            for (int u = unit_seq(cta, 0, G, p.unit_run); ok && u < n_units; ++it, u = unit_seq(cta, it, G, p.unit_run)) {
                const Unit x = decode_unit<SPLIT, MOD, D == 64>(p, u, kv_next, false);
                kv_next = unit_key_len<D == 64>(p, unit_seq(cta, it + 1, G, p.unit_run), n_units);
                const int qb = it % QS;
                const int n_max = x.n_max();
                if (n_max == 0) continue;  // nothing to load; its epilogue does not use a Q buffer
                // the Q buffer is free once both tiles' stores of its previous unit have read it
                if (q_loads[qb] > 0 &&
                    !mbar_wait(bar(L::QEMPTY + qb), (q_loads[qb] - 1) & 1, limit, abort_flag, p.epoch, kRoleProducer, 9))
                    { ok = false; break; }
                const int n_q_tiles = x.tile_b_valid ? 2 : 1;
                mbar_arrive_expect_tx(bar(L::QFULL + qb), n_q_tiles * L::kTileBytes);
                for (int t = 0; t < n_q_tiles; ++t) {
                    #pragma unroll
                    for (int c = 0; c < L::kChunks; ++c)
                        tma_load_3d(sbase + L::kQ + qb * L::kQBuf + t * L::kTileBytes + c * L::kChunkBytes, &tm_q,
                                    bar(L::QFULL + qb), c * kElemsPerChunk, x.q0 + t * kBM, x.bh);
                }
                ++q_loads[qb];
                for (int i = 0; i < 2 * n_max; ++i, ++i_glob) {  // K_0, V_0, K_1, V_1, ...
                    const int s = i_glob % NSLOT;
                    const int use = i_glob / NSLOT;
                    if (use > 0 &&
                        !mbar_wait(bar(L::EMPTY + s), (use - 1) & 1, limit, abort_flag, p.epoch, kRoleProducer, 10))
                        { ok = false; break; }
                    const CUtensorMap* map = (i & 1) ? &tm_v : &tm_k;
                    mbar_arrive_expect_tx(bar(L::FULL + s), L::kTileBytes);
                    #pragma unroll
                    for (int c = 0; c < L::kChunks; ++c)
                        tma_load_3d(sbase + L::kRing + s * L::kTileBytes + c * L::kChunkBytes, map, bar(L::FULL + s),
                                    c * kElemsPerChunk, (x.j_lo + (i >> 1)) * kBN, x.bhk);
                    uses[s] = use + 1;
                }
            }
            // Drain: every load this thread issued has landed before the CTA may exit.
            #pragma unroll
            for (int q = 0; q < QS; ++q)
                if (q_loads[q] > 0) mbar_drain(bar(L::QFULL + q), (q_loads[q] - 1) & 1, kRoleProducer, 12);
            #pragma unroll
            for (int s = 0; s < NSLOT; ++s)
                if (uses[s] > 0) mbar_drain(bar(L::FULL + s), (uses[s] - 1) & 1, kRoleProducer, 13);
        }
      } else {
        // =============================== MMA issuer ===============================
        // The whole warp runs this loop (warp-uniform control flow and operands);
        // one elected lane issues each tcgen05 instruction.  Decoupled S and P:
        // warp 9 serves tile A and warp 10 tile B, each with waits of its own.
        {
            const int mt = kDec ? warp - 9 : 0;
            constexpr uint32_t kIdescS = FP8 ? idesc_e4m3_f32(kBM, kBN, false) : idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t kIdescO = FP8 ? idesc_e4m3_f32(kBM, D, true) : idesc_bf16_f32(kBM, D, true);
            // K steps of one MMA: 16 bf16 or 32 FP8 elements, 32 bytes either way
            constexpr int kSSteps = FP8 ? D / 32 : D / 16;
            constexpr int kPvKeys = FP8 ? 32 : 16;          // keys per PV step
            constexpr int kPvSteps = (kBN / 2) / kPvKeys;   // per half of P
            int q_loads[QS];
            #pragma unroll
            for (int q = 0; q < QS; ++q) q_loads[q] = 0;
            int i_glob = 0;      // K/V loads consumed so far
            int gp[2] = {0, 0};  // P_t blocks consumed so far (P0 / P1 phase)
            int gf[2] = {0, 0};  // SFREE_t phases waited for (decoupled S and P)
            bool ok = true;
            int it = 0;
            int kv_next = unit_key_len<D == 64>(p, unit_seq(cta, 0, G, p.unit_run), n_units);
            for (int u = unit_seq(cta, 0, G, p.unit_run); ok && u < n_units; ++it, u = unit_seq(cta, it, G, p.unit_run)) {
                const Unit x = decode_unit<SPLIT, MOD, D == 64>(p, u, kv_next, false);
                kv_next = unit_key_len<D == 64>(p, unit_seq(cta, it + 1, G, p.unit_run), n_units);
                const int n_max = x.n_max();
                if (n_max == 0) continue;
                const int qb = it % QS;
                const uint32_t qbuf = sbase + L::kQ + qb * L::kQBuf;
                auto slot_of = [&](int i) { return (i_glob + i) % NSLOT; };
                auto wait_full = [&](int i, unsigned site) -> bool {
                    return mbar_wait_warp(bar(L::FULL + slot_of(i)), ((i_glob + i) / NSLOT) & 1, limit, abort_flag,
                                     p.epoch, kRoleMma, site);
                };
                // S_t(j) = Q_t K_j^T in batches of four K steps (32 bytes each), then the
                // SFULL_t commit and an optional second commit (0: none)
                auto issue_s = [&](int t, int j, uint32_t bar_b = 0u) {
                    const uint64_t qd = smem_desc_sw128(qbuf + t * L::kTileBytes, 16, 1024);
                    const uint64_t kd = smem_desc_sw128(sbase + L::kRing + slot_of(2 * j) * L::kTileBytes, 16, 1024);
                    static_assert(kSSteps == 4 || kSSteps == 8, "S steps");
                    #pragma unroll
                    for (int g = 0; g < kSSteps / 4; ++g) {
                        const uint64_t o = static_cast<uint64_t>(g * (L::kChunkBytes >> 4));  // descriptor units
                        const bool last = g == kSSteps / 4 - 1;
                        mma_ss_batch_warp<FP8, 4, 2, 2>(tmem + t * 128, qd + o, kd + o, kIdescS, g > 0 ? 1u : 0u,
                                                        last ? bar(L::SFULL + t) : 0u, last ? bar_b : 0u);
                    }
                };
                // O_t += P_t(j)[:, keys of this half] V_j[those keys, :], then up to two commits
                auto issue_pv = [&](int t, int j, int half, uint32_t bar_a = 0u, uint32_t bar_b = 0u) {
                    const uint32_t v_addr = sbase + L::kRing + slot_of(2 * j + 1) * L::kTileBytes;
                    const uint32_t o_tmem = tmem + L::kColO + t * D;
                    const int kk0 = half * kPvSteps;
                    const uint64_t vd = smem_desc_sw128(v_addr + kk0 * kPvKeys * 128, L::kChunkBytes, 1024);
                    constexpr uint64_t kVStep = kPvKeys * 128 / 16;  // one step of keys, descriptor units
                    const uint32_t acc0 = (j > 0 || kk0 > 0) ? 1u : 0u;
                    if constexpr (FP8) {
                        // P_t in shared memory, 128-byte K-major rows (SW128), 32 keys per step
                        static_assert(kPvSteps == 2, "PV steps");
                        const uint64_t pd = smem_desc_sw128(sbase + L::kPS + t * L::kPBytes + kk0 * 32, 16, 1024);
                        mma_ss_batch_warp<true, 2, 2, static_cast<int>(kVStep)>(o_tmem, pd, vd, kIdescO, acc0, bar_a,
                                                                                bar_b);
                    } else {
                        static_assert(kPvSteps == 4, "PV steps");
                        const uint32_t pt = (kDec ? tmem + L::kColP + t * 64 : tmem + t * 128) + kk0 * 8;
                        mma_ts4_batch_warp<8, static_cast<int>(kVStep)>(o_tmem, pt, vd, kIdescO, acc0, bar_a, bar_b);
                    }
                };
                ok = mbar_wait_warp(bar(L::QFULL + qb), q_loads[qb] & 1, limit, abort_flag, p.epoch, kRoleMma, 20) &&
                     wait_full(0, 21);
                ++q_loads[qb];
                if (!ok) break;
                tc_fence_after();
                if constexpr (kDec) {
                    // One tile: S_t(j+1) as soon as the softmax has read S_t(j) (SFREE),
                    // then PV_t(j) by halves as P_t(j) is stored (P0, P1).  Every K/V load
                    // of the unit is released once by each of the two warps: after the
                    // products that read it, or, for blocks this tile does not use, once
                    // the load has landed (so that the arrival cannot count towards the
                    // slot's previous use).
                    const int t = mt;
                    const int nt = x.n_t[t];
                    auto release_unused = [&](int i, unsigned site) -> bool {
                        if (!wait_full(i, site)) return false;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(L::EMPTY + slot_of(i)));
                        return true;
                    };
                    if (nt > 0) {
                        issue_s(t, 0, bar(L::EMPTY + slot_of(0)));  // and K_0 released
                    } else {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(L::EMPTY + slot_of(0)));
                    }
                    for (int j = 0; ok && j < nt; ++j) {
                        if (j + 1 < nt) {
                            if (!mbar_wait_warp(bar(L::SFREE + t), gf[t] & 1, limit, abort_flag, p.epoch, kRoleMma, 28) ||
                                !wait_full(2 * j + 2, 29))
                                { ok = false; break; }
                            ++gf[t];
                            tc_fence_after();
                            issue_s(t, j + 1, bar(L::EMPTY + slot_of(2 * j + 2)));  // and K_{j+1} released
                        }
                        if (!mbar_wait_warp(bar(L::P0 + t), gp[t] & 1, limit, abort_flag, p.epoch, kRoleMma, 22))
                            { ok = false; break; }
                        if (j == 0 && it > 0 &&
                            !mbar_wait_warp(bar(L::OEMPTY + t), (it - 1) & 1, limit, abort_flag, p.epoch, kRoleMma, 23))
                            { ok = false; break; }
                        if (!wait_full(2 * j + 1, 24)) { ok = false; break; }
                        tc_fence_after();
                        issue_pv(t, j, 0);
                        if (!mbar_wait_warp(bar(L::P1 + t), gp[t] & 1, limit, abort_flag, p.epoch, kRoleMma, 27))
                            { ok = false; break; }
                        ++gp[t];
                        tc_fence_after();
                        // then PVDONE_t (OFINAL_t after the last block) and V_j released
                        issue_pv(t, j, 1, bar((j + 1 < nt ? L::PVDONE : L::OFINAL) + t), bar(L::EMPTY + slot_of(2 * j + 1)));
                    }
                    // loads of the unit past this tile's last block, in load order
                    for (int j = nt; ok && j < n_max; ++j) {
                        if (j > 0 && !release_unused(2 * j, 36)) { ok = false; break; }
                        if (!release_unused(2 * j + 1, 37)) { ok = false; break; }
                    }
                } else {
                for (int t = 0; t < 2; ++t)
                    if (x.n_t[t] > 0) issue_s(t, 0);
                mma_commit_warp(bar(L::EMPTY + slot_of(0)));  // K_0 released once both S(0) complete
                for (int j = 0; ok && j < n_max; ++j) {
                    bool v_ready = false, k_next_ready = false;
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (j >= x.n_t[t]) continue;
                        // first half of P_t(j): PV over keys 0..63 overlaps the rest of the softmax
                        if (!mbar_wait_warp(bar(L::P0 + t), gp[t] & 1, limit, abort_flag, p.epoch, kRoleMma, 22))
                            { ok = false; break; }
                        // the previous unit's epilogue must have read O_t out of TMEM
                        if (j == 0 && it > 0 &&
                            !mbar_wait_warp(bar(L::OEMPTY + t), (it - 1) & 1, limit, abort_flag, p.epoch, kRoleMma, 23))
                            { ok = false; break; }
                        if (!v_ready) {
                            if (!wait_full(2 * j + 1, 24)) { ok = false; break; }
                            v_ready = true;
                        }
                        tc_fence_after();
                        issue_pv(t, j, 0);
                        if (!mbar_wait_warp(bar(L::P1 + t), gp[t] & 1, limit, abort_flag, p.epoch, kRoleMma, 27))
                            { ok = false; break; }
                        ++gp[t];
                        tc_fence_after();
                        const bool last_t = j + 1 >= x.n_t[t];
                        issue_pv(t, j, 1, last_t ? bar(L::OFINAL + t) : 0u);
                        if (!last_t) {
                            if (!k_next_ready) {
                                if (!wait_full(2 * j + 2, 25)) { ok = false; break; }
                                k_next_ready = true;
                                tc_fence_after();
                            }
                            issue_s(t, j + 1);
                        }
                    }
                    if (!ok) break;
                    // V_j (both PV(j) issued above) and K_{j+1}: the tile with n_t = n_max uses
                    // every block, so k_next_ready holds exactly when j + 1 < n_max (each load
                    // is released once).
                    mma_commit2_warp(bar(L::EMPTY + slot_of(2 * j + 1)),
                                     k_next_ready ? bar(L::EMPTY + slot_of(2 * j + 2)) : 0u);
                }
                }
                i_glob += 2 * n_max;
            }
            mma_commit_warp(bar(L::MMAFIN));
            mbar_drain(bar(L::MMAFIN), 0, kRoleMma, 26);
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(kRegsSoftmax));
        // =================== softmax + epilogue warpgroups (tiles A, B) ===================
        const int t = warp >> 2;  // tile
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_tmem = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t s_tmem = lane_tmem + t * 128;
        const uint32_t o_tmem = lane_tmem + L::kColO + t * D;
        const float c_log2 = p.scale_log2;
        const uint64_t c2 = pack_f32x2(c_log2, c_log2);
        int gs = 0;       // S_t blocks consumed so far (SFULL phase)
        int gpd = 0;      // PVDONE_t phases waited for (decoupled S and P)
        int n_final = 0;  // units with a PV for this tile so far (OFINAL phase)
        bool ok = true;
        int it = 0;
        int kv_next = unit_key_len<D == 64>(p, unit_seq(cta, 0, G, p.unit_run), n_units);
        for (int u = unit_seq(cta, 0, G, p.unit_run); u < n_units; ++it, u = unit_seq(cta, it, G, p.unit_run)) {
            const Unit x = decode_unit<SPLIT, MOD, D == 64>(p, u, kv_next, threadIdx.x == 0);
            kv_next = unit_key_len<D == 64>(p, unit_seq(cta, it + 1, G, p.unit_run), n_units);
            const int q0_t = x.q0 + t * kBM;
            const int q_idx = q0_t + row;
            const int n_blocks = ok ? x.n_t[t] : 0;
            const int kv_len = x.kv_len;
            float m_used = -INFINITY;  // running max (base-2, scaled), possibly stale by < tau
            float l_sum = 0.0f;        // running sum of exp2(t - m_used)
            Rect2D rq{0, 0, 0, 0};
            if constexpr (MOD) {
                if (p.m2_kind != 0) rq = rect_2d(p, q_idx);
            }
            // FP8: this tile's Q block scale and the largest V block scale of the head
            // (P is stored as 2^6 * P * sv_block / sv_max so that one O accumulator
            // serves every key block; O is multiplied by 2^-6 sv_max at the end)
            float sq_t = 1.0f, sv_max = 1.0f;
            if constexpr (FP8) {
                if (q0_t < p.Nq) sq_t = __ldg(p.q_scale + static_cast<long long>(x.bh) * p.nqb + q0_t / kBM);
                const float* vsr = p.v_scale + static_cast<long long>(x.bhk) * p.nkb;
                sv_max = 0.0f;
                for (int i = 0; i < p.nkb; ++i) sv_max = fmaxf(sv_max, __ldg(vsr + i));
                if (!(sv_max > 0.0f)) sv_max = 1.0f;
            }
            const float* mask_row = nullptr;
            if constexpr (HAS_MASK) {
                if (q_idx < p.Nq)
                    mask_row = p.mask + static_cast<long long>(x.b) * p.msb + static_cast<long long>(x.h) * p.msh +
                               static_cast<long long>(q_idx) * p.msq;
            }

            // FP8: the K and V block scales of the next key block, loaded one block ahead
            const long long kb0 = static_cast<long long>(x.bhk) * p.nkb + x.j_lo;
            float ks_next = 1.0f, vs_next = 1.0f;
            if constexpr (FP8) {
                if (n_blocks > 0) {
                    ks_next = __ldg(p.k_scale + kb0);
                    vs_next = __ldg(p.v_scale + kb0);
                }
            }
            for (int j = 0; j < n_blocks; ++j) {
                const float ksb = ks_next, svb = vs_next;
                if constexpr (FP8) {
                    if (j + 1 < n_blocks) {
                        ks_next = __ldg(p.k_scale + kb0 + j + 1);
                        vs_next = __ldg(p.v_scale + kb0 + j + 1);
                    }
                }
                bool got = mbar_wait(bar(L::SFULL + t), gs & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 30);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                ++gs;
                tc_fence_after();
                uint32_t sr[kBN];
                #pragma unroll
                for (int c = 0; c < kBN / 32; ++c)
                    tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
                tmem_wait_ld();
                if constexpr (kDec) {
                    // S_t(j) is in registers: the MMA warp may overwrite it with S_t(j+1)
                    if (j + 1 < n_blocks) {
                        tc_fence_before();
                        mbar_arrive(bar(L::SFREE + t));
                    }
                }
                float* s = reinterpret_cast<float*>(sr);
                const int j0 = (x.j_lo + j) * kBN;
                const bool boundary = (j0 + kBN > kv_len) || (p.is_causal && j0 + kBN - 1 > q0_t);
                // score scale of this block (FP8: times the Q and K block scales) and, for
                // FP8, log2 of this block's V scale relative to the head's largest
                float cl = c_log2, lr = 0.0f, inv_r = 1.0f;
                if constexpr (FP8) {
                    cl = c_log2 * sq_t * ksb;
                    lr = svb > 0.0f ? __log2f(svb / sv_max) + kPShiftF8 : -INFINITY;
                    inv_r = svb > 0.0f ? sv_max / svb * exp2f(-kPShiftF8) : 0.0f;
                }
                const uint64_t cl2 = pack_f32x2(cl, cl);

                // keys c >= lim of this block are masked (padding / past the diagonal)
                int lim = kv_len - j0;
                if (p.is_causal && q_idx - j0 + 1 < lim) lim = q_idx - j0 + 1;
                if constexpr (MOD) {
                    if (p.softcap_on) {
                        // base-2 logit cap * log2(e) * tanh(x / cap).  When every raw score
                        // of the warp's block has |scale * s / cap| <= kTanhPolyRange, tanh is
                        // the odd polynomial (FMA pipe only); otherwise tanh(u) =
                        // 1 - 2 / (1 + e^(2u)) on the special-function unit.
                        float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
                        #pragma unroll
                        for (int c = 0; c < kBN; c += 8) {
                            a0 = fmax3(a0, fabsf(s[c]), fabsf(s[c + 1]));
                            a1 = fmax3(a1, fabsf(s[c + 2]), fabsf(s[c + 3]));
                            a2 = fmax3(a2, fabsf(s[c + 4]), fabsf(s[c + 5]));
                            a3 = fmax3(a3, fabsf(s[c + 6]), fabsf(s[c + 7]));
                        }
                        const bool in_range = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) <= p.sc_lim;
                        if (__all_sync(0xffffffffu, in_range)) {
                            const uint64_t ca = pack_f32x2(p.sc_a, p.sc_a);
                            #pragma unroll
                            for (int c = 0; c < kBN / 2; ++c) {
                                const uint64_t sv = pack_f32x2(s[2 * c], s[2 * c + 1]);
                                const uint64_t t = ffma2(sv, ca, 0ull);
                                const uint64_t w = ffma2(t, t, 0ull);
                                uint64_t h = ffma2(w, pack_f32x2(p.sc_poly[5], p.sc_poly[5]),
                                                   pack_f32x2(p.sc_poly[4], p.sc_poly[4]));
                                h = ffma2(w, h, pack_f32x2(p.sc_poly[3], p.sc_poly[3]));
                                h = ffma2(w, h, pack_f32x2(p.sc_poly[2], p.sc_poly[2]));
                                h = ffma2(w, h, pack_f32x2(p.sc_poly[1], p.sc_poly[1]));
                                h = ffma2(w, h, pack_f32x2(p.sc_poly[0], p.sc_poly[0]));
                                const uint64_t r = ffma2(sv, h, 0ull);
                                s[2 * c] = lo_f32(r);
                                s[2 * c + 1] = hi_f32(r);
                            }
                        } else {
                            #pragma unroll
                            for (int c = 0; c < kBN; ++c)
                                s[c] = fmaf(rcp_approx(1.0f + ex2_approx(s[c] * p.sc_in)), -2.0f * p.sc_out, p.sc_out);
                        }
                    }
                    if (p.m2_kind != 0) {
                        // keys of this block inside the row's grid rectangle, as a 128-bit set:
                        // one run of columns per key row the block touches
                        uint32_t mw[kBN / 32] = {0u, 0u, 0u, 0u};
                        const int W = p.m2_w;
                        int kr = fdiv(j0, p.fd_w);
                        const int kr_end = fdiv(j0 + kBN - 1, p.fd_w);
                        if (kr < rq.r_lo) kr = rq.r_lo;
                        for (; kr <= kr_end && kr <= rq.r_hi; ++kr) {
                            int a = kr * W + rq.c_lo - j0, b = kr * W + rq.c_hi - j0;
                            if (a < 0) a = 0;
                            if (b > kBN - 1) b = kBN - 1;
                            #pragma unroll
                            for (int w = 0; w < kBN / 32; ++w) {
                                const int lo = a - 32 * w > 0 ? a - 32 * w : 0;
                                const int hi = b - 32 * w < 31 ? b - 32 * w : 31;
                                if (lo <= hi) mw[w] |= ((2u << (hi - lo)) - 1u) << lo;
                            }
                        }
                        #pragma unroll
                        for (int c = 0; c < kBN; ++c)
                            s[c] = (((mw[c >> 5] >> (c & 31)) & 1u) && c < lim) ? s[c] : -INFINITY;
                    } else if (boundary) {
                        #pragma unroll
                        for (int c = 0; c < kBN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
                    }
                } else if constexpr (!HAS_MASK) {
                    if (boundary) {
                        // one compare and select per element, c a compile-time constant
                        #pragma unroll
                        for (int c = 0; c < kBN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
                    }
                }
                // exponent arguments and exponentials of keys [64h, 64h + 64) in place
                auto exp_keys = [&](auto half_c, uint64_t ns2) {
                    constexpr int kN = kBN / 2;
                    float* sh = s + decltype(half_c)::value * kN;
                    if constexpr (HAS_MASK) {
                        const float sft = -lo_f32(ns2);
                        #pragma unroll
                        for (int c = 0; c < kN; ++c) sh[c] = ex2_approx(sh[c] - sft);
                    } else {
                        constexpr int kEmu = FP8 ? ATTN_F8_EXP_EMU : 0;
                        #pragma unroll
                        for (int c = 0; c < kN / 2; ++c) {
                            const uint64_t xv = ffma2(pack_f32x2(sh[2 * c], sh[2 * c + 1]), cl2, ns2);
                            if (kEmu > 0 && c % (kEmu > 0 ? kEmu : 1) == kEmu - 1) {
                                const uint64_t r = exp2_poly_x2(xv);
                                sh[2 * c] = lo_f32(r);
                                sh[2 * c + 1] = hi_f32(r);
                            } else {
                                sh[2 * c] = ex2_approx(lo_f32(xv));
                                sh[2 * c + 1] = ex2_approx(hi_f32(xv));
                            }
                        }
                    }
                };
                auto row_max = [&]() -> float {
                    float m0 = fmax3(s[0], s[1], s[2]), m1 = fmax3(s[3], s[4], s[5]);
                    float m2 = fmax3(s[6], s[7], s[8]), m3 = fmax3(s[9], s[10], s[11]);
                    #pragma unroll
                    for (int c = 12; c + 7 < kBN; c += 8) {
                        m0 = fmax3(m0, s[c], s[c + 1]);
                        m1 = fmax3(m1, s[c + 2], s[c + 3]);
                        m2 = fmax3(m2, s[c + 4], s[c + 5]);
                        m3 = fmax3(m3, s[c + 6], s[c + 7]);
                    }
                    m0 = fmax3(m0, s[kBN - 4], s[kBN - 3]);
                    m1 = fmax3(m1, s[kBN - 2], s[kBN - 1]);
                    return fmax3(m0, m1, fmaxf(m2, m3));
                };

                float mx;
                if constexpr (HAS_MASK) {
                    mx = -INFINITY;
                    const int mlim = mask_row != nullptr ? lim : 0;
                    #pragma unroll
                    for (int c = 0; c < kBN; ++c) {
                        const bool valid = c < mlim;
                        const float mv = valid ? __ldg(mask_row + j0 + c) : 0.0f;
                        s[c] = valid ? fmaf(s[c], c_log2, mv * kLog2e) : -INFINITY;
                        mx = fmaxf(mx, s[c]);
                    }
                } else {
                    mx = row_max() * cl;
                }

                // Lazy correction, decided per row: a row moves its reference max only when
                // the block max exceeds it by more than tau.  The TMEM load/store of O_t is
                // warp-collective, but rows that keep their max use alpha = 1 exactly, so a
                // row's result never depends on the other rows of its warp.  O_t holds
                // sum_{i<j} P_i V_i here (S_t(j) was issued after PV_t(j-1)); the rescale
                // of O_t itself is done after the first half of P_t is stored (fewer live
                // registers) and before the P0 arrive that lets PV_t(j) start.
                const bool need = mx > m_used + (FP8 ? kLazyTauF8 : kLazyTau);
                const bool warp_rescale = __any_sync(0xffffffffu, need) && j > 0;
                float alpha = 1.0f;
                if (need) {
                    alpha = (m_used == -INFINITY) ? 0.0f : ex2_approx(m_used - mx);
                    l_sum *= alpha;
                    m_used = mx;
                }
                const float shift = (m_used == -INFINITY) ? 0.0f : m_used;
                const uint64_t nshift2 = pack_f32x2(lr - shift, lr - shift);

                uint64_t acc0 = 0, acc1 = 0, acc2 = 0, acc3 = 0;  // packed partial sums
                uint32_t pk[FP8 ? kBN / 8 : kBN / 4];
                // row-sum terms and bf16 pairs of keys [64h, 64h + 64)
                auto pack_half = [&](auto half_c) {
                    float* sh = s + decltype(half_c)::value * (kBN / 2);
                    #pragma unroll
                    for (int c = 0; c < kBN / 4; ++c) {
                        const uint64_t e = pack_f32x2(sh[2 * c], sh[2 * c + 1]);
                        switch (c & 3) {
                            case 0: acc0 = fadd2(acc0, e); break;
                            case 1: acc1 = fadd2(acc1, e); break;
                            case 2: acc2 = fadd2(acc2, e); break;
                            default: acc3 = fadd2(acc3, e); break;
                        }
                        if constexpr (FP8) {
                            if ((c & 1) == 0)
                                pk[c >> 1] = pack_e4m3x4(sh[2 * c], sh[2 * c + 1], sh[2 * c + 2], sh[2 * c + 3]);
                        } else {
                            pk[c] = pack_bf16x2(sh[2 * c], sh[2 * c + 1]);
                        }
                    }
                };
                exp_keys(std::integral_constant<int, 0>{}, nshift2);
                pack_half(std::integral_constant<int, 0>{});

                // Keys 0..63, then 64..127: each half is stored and signalled on its own
                // (P0, P1), so PV over the first half runs during the second half.  O_t is
                // rescaled (if needed) before P0 releases the first PV.
                auto store_half = [&](auto half_c) -> bool {
                    constexpr int h = decltype(half_c)::value;
                    if constexpr (kDec) {
                        // PV_t(j-1) must be complete before P_t and O_t are touched
                        if (h == 0 && j > 0) {
                            const bool got_pv = mbar_wait(bar(L::PVDONE + t), gpd & 1, limit, abort_flag, p.epoch,
                                                          kRoleSoftmax, 33);
                            ++gpd;
                            if (!__all_sync(0xffffffffu, got_pv)) return false;
                            tc_fence_after();
                        }
                    }
                    if constexpr (FP8) {
                        // 64 keys = 64 bytes of this row, four 16-byte units at swizzled positions
                        const uint32_t prow = sbase + L::kPS + t * L::kPBytes + row * 128;
                        #pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            st_shared_v4(prow + (((h * 4 + c4) ^ (row & 7)) << 4), pk[4 * c4], pk[4 * c4 + 1],
                                         pk[4 * c4 + 2], pk[4 * c4 + 3]);
                        fence_proxy_async_smem();
                    } else if constexpr (kDec) {
                        tmem_st32(lane_tmem + L::kColP + t * 64 + h * 32, pk);
                    } else {
                        tmem_st32(s_tmem + h * 32, pk);
                    }
                    if (h == 0 && warp_rescale) {
                        #pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(o_tmem + c * 32, o);
                            tmem_wait_ld();
                            #pragma unroll
                            for (int v = 0; v < 32; ++v) o[v] = __float_as_uint(__uint_as_float(o[v]) * alpha);
                            tmem_st32(o_tmem + c * 32, o);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar((h == 0 ? L::P0 : L::P1) + t));
                    return true;
                };
                if (!store_half(std::integral_constant<int, 0>{})) { ok = false; break; }
                exp_keys(std::integral_constant<int, 1>{}, nshift2);
                pack_half(std::integral_constant<int, 1>{});
                store_half(std::integral_constant<int, 1>{});
                const uint64_t acc = fadd2(fadd2(acc0, acc2), fadd2(acc1, acc3));
                l_sum += (lo_f32(acc) + hi_f32(acc)) * inv_r;
            }

            // ------------------------------------------------------------ epilogue
            const int qb = it % QS;
            // QEMPTY expects two arrivals per loaded unit.  Only a tile with key blocks
            // arrives (on behalf of both when the other tile has none): a tile without
            // work waits on nothing, so its arrivals could run ahead into a later
            // unit's phase of the barrier.
            auto release_q = [&](int b) {
                if (x.n_t[t] > 0) mbar_arrive_cnt(bar(L::QEMPTY + b), x.n_t[t ^ 1] > 0 ? 1u : 2u);
            };
            if (x.n_max() == 0) {
                // No unmasked key at all (key length 0): O = 0, LSE = -inf, written
                // directly (this unit loaded nothing and owns no Q buffer).
                tc_fence_before();
                mbar_arrive(bar(L::OEMPTY + t));
                if (q_idx < p.Nq && (t == 0 || x.tile_b_valid) && ok && !*abort_flag) {
                    const long long r = static_cast<long long>(x.bh) * p.Nq + q_idx;
                    if constexpr (SPLIT) {
                        const long long rs = static_cast<long long>(x.split) * p.B * p.Hq * p.Nq + r;
                        float4* dst = reinterpret_cast<float4*>(p.ws_o + rs * D);
                        #pragma unroll
                        for (int v = 0; v < D / 4; ++v) dst[v] = make_float4(0.f, 0.f, 0.f, 0.f);
                        p.ws_lse[rs] = -INFINITY;
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + r * D);
                        #pragma unroll
                        for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                        if (p.lse != nullptr) p.lse[r] = -INFINITY;
                    }
                }
                continue;
            }
            if (ok && n_blocks > 0) {
                bool got = mbar_wait(bar(L::OFINAL + t), n_final & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 32);
                ok = __all_sync(0xffffffffu, got);
                ++n_final;
                tc_fence_after();
            }
            // Q_t has been read by every S_t of the unit (OFINAL_t).  Unless O is staged
            // in it (bf16, d = 128), the producer may refill the Q buffer now.
            constexpr bool kOStage = !SPLIT && !FP8 && D == 64;  // bf16 O staged in a buffer of its own
            if constexpr (SPLIT || FP8 || kOStage) {
                if ((threadIdx.x & 127) == 0) release_q(qb);
            }
            // (tile B of a single-tile unit writes nothing: its rows belong to the unit's
            // other half, whose own unit computes them)
            const bool do_epilogue = __all_sync(0xffffffffu, ok && !*abort_flag) && q0_t < p.Nq &&
                                     (t == 0 || x.tile_b_valid);
            const float inv_l = l_sum > 0.0f ? 1.0f / l_sum : 0.0f;
            if constexpr (SPLIT) {
                // Split-KV: this key range's O (normalised by its own row sum) and LSE go
                // to the workspace in fp32, row by row; the combine kernel merges them.
                const long long rs = (static_cast<long long>(x.split) * p.B * p.Hq + x.bh) * p.Nq + q_idx;
                #pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    if (n_blocks > 0 && do_epilogue) {
                        tmem_ld32(o_tmem + c * 32, o);
                        tmem_wait_ld();
                    } else {
                        #pragma unroll
                        for (int v = 0; v < 32; ++v) o[v] = 0u;
                    }
                    if (c == D / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(bar(L::OEMPTY + t));
                    }
                    if (do_epilogue && q_idx < p.Nq) {
                        float4* dst = reinterpret_cast<float4*>(p.ws_o + rs * D + c * 32);
                        #pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                                 __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
                    }
                }
                if (do_epilogue && q_idx < p.Nq)
                    p.ws_lse[rs] = l_sum > 0.0f ? (m_used + __log2f(l_sum)) * kLn2 : -INFINITY;
            } else if constexpr (FP8) {
                // O = 2^-6 sv_max acc / l, bf16, each thread writing its own row straight
                // from registers (the FP8 Q buffer is too small to stage bf16 tiles)
                const float scl = inv_l * sv_max * exp2f(-kPShiftF8);
                uint16_t* orow = static_cast<uint16_t*>(p.out) + (static_cast<long long>(x.bh) * p.Nq + q_idx) * D;
                #pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    if (n_blocks > 0 && do_epilogue) {
                        tmem_ld32(o_tmem + c * 32, o);
                        tmem_wait_ld();
                    } else {
                        #pragma unroll
                        for (int v = 0; v < 32; ++v) o[v] = 0u;
                    }
                    if (c == D / 32 - 1) {
                        // O_t has been read out of TMEM: the next unit's PV_t(0) may overwrite it.
                        tc_fence_before();
                        mbar_arrive(bar(L::OEMPTY + t));
                    }
                    if (do_epilogue && q_idx < p.Nq) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
                        #pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(
                                pack_bf16x2(__uint_as_float(o[8 * v]) * scl, __uint_as_float(o[8 * v + 1]) * scl),
                                pack_bf16x2(__uint_as_float(o[8 * v + 2]) * scl, __uint_as_float(o[8 * v + 3]) * scl),
                                pack_bf16x2(__uint_as_float(o[8 * v + 4]) * scl, __uint_as_float(o[8 * v + 5]) * scl),
                                pack_bf16x2(__uint_as_float(o[8 * v + 6]) * scl, __uint_as_float(o[8 * v + 7]) * scl));
                    }
                }
                if (do_epilogue && q_idx < p.Nq && p.lse != nullptr)
                    p.lse[static_cast<long long>(x.bh) * p.Nq + q_idx] =
                        l_sum > 0.0f ? (m_used + __log2f(l_sum)) * kLn2 : -INFINITY;
            } else {
            // bf16 O through shared memory (128-byte swizzled rows) and one TMA store per
            // tile.  d = 64: a staging buffer of its own, whose previous store is waited
            // for here, a unit later; d = 128: the dead Q_t buffer, released once the
            // store has read it.
            uint8_t* stage = kOStage ? smem + L::kOS + t * L::kTileBytes
                                     : smem + L::kQ + qb * L::kQBuf + t * L::kTileBytes;
            if constexpr (kOStage) {
                if ((threadIdx.x & 127) == 0) bulk_wait_group_read0();
                named_barrier_sync(1 + t, 128);
            }
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (n_blocks > 0 && do_epilogue) {
                    tmem_ld32(o_tmem + c * 32, o);
                    tmem_wait_ld();
                } else {
                    #pragma unroll
                    for (int v = 0; v < 32; ++v) o[v] = 0u;
                }
                if (c == D / 32 - 1) {
                    // O_t has been read out of TMEM: the next unit's PV_t(0) may overwrite it.
                    tc_fence_before();
                    mbar_arrive(bar(L::OEMPTY + t));
                }
                if (do_epilogue) {
                    uint32_t w[16];
                    #pragma unroll
                    for (int v = 0; v < 16; ++v)
                        w[v] = pack_bf16x2(__uint_as_float(o[2 * v]) * inv_l, __uint_as_float(o[2 * v + 1]) * inv_l);
                    const int chunk = (c * 32) / 64;
                    const int unit0 = ((c * 32) % 64) / 8;
                    #pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int phys = (unit0 + v) ^ (row & 7);
                        uint4* dst = reinterpret_cast<uint4*>(stage + chunk * L::kChunkBytes + row * 128 + phys * 16);
                        *dst = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                    }
                }
            }
            if (do_epilogue) {
                fence_proxy_async_smem();
                if (p.lse != nullptr && q_idx < p.Nq) {
                    const float lse = l_sum > 0.0f ? (m_used + __log2f(l_sum)) * kLn2 : -INFINITY;
                    p.lse[static_cast<long long>(x.bh) * p.Nq + q_idx] = lse;
                }
            }
            named_barrier_sync(1 + t, 128);
            if ((threadIdx.x & 127) == 0) {
                if (do_epilogue && !*abort_flag) {
                    #pragma unroll
                    for (int c = 0; c < L::kChunks; ++c)
                        tma_store_3d(&tm_o, smem_u32(stage) + c * L::kChunkBytes, c * 64, q0_t, x.bh);
                    bulk_commit_group();
                    if constexpr (!kOStage) bulk_wait_group_read0();
                }
                if constexpr (!kOStage) release_q(qb);  // the producer may refill this Q buffer
            }
            }  // !SPLIT
        }
    }

    // ================================ teardown ================================
    // (a TMA store still reading the O staging buffer must finish before the CTA exits)
    if (warp < 8 && (threadIdx.x & 127) == 0) bulk_wait_group_read0();
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn_sm100
