// bwd_kernels.cuh -- backward pass of exact attention for sm_100a.
//
// "FlashAttention technical analysis" (jsqmd.com/news/722897), section 3.3:
// the forward pass keeps only O(N) statistics per row (here the LSE); the
// backward pass recomputes each block of P from Q, K and those statistics
// instead of reading a stored N x N matrix.  With S = scale * Q K^T,
// P = exp(S - LSE), D_i = sum_t dO_it O_it:
//
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - D),   dQ = scale dS K,   dK = scale dS^T Q
//
// Three launches:
//   attn_bwd_prep_kernel         D and LSE * log2(e) per query row (HBM-bound, a warp per row)
//   attn_bwd_kernel<D, true>     dK, dV: one CTA per 128-key block of one K/V head, looping
//                                over the query blocks of every query head of its group (K/V
//                                blocks in the outer loop, section 4.1 of the same page);
//                                S^T = K Q^T and dP^T = V dO^T on the tensor cores, P^T and
//                                dS^T written back to TMEM as bf16, then dV += P^T dO and
//                                dK += dS^T Q accumulate in TMEM
//   attn_bwd_kernel<D, false>    dQ: one CTA per 128-row query block, looping over key
//                                blocks; S = Q K^T, dP = dO V^T, dS to TMEM, dQ += dS K
// Splitting dQ from dK/dV keeps every accumulator in one CTA's TMEM: no atomics.
// Each iteration's 128 columns pass in two halves of 64 through two TMEM buffers,
// so that the elementwise step of one half overlaps the tensor work of its
// neighbours (the accumulating products of the previous half, S and dP of the
// next).
//
// Score and mask variants (the VAR instantiation), the forward's readings: the
// score is s = c(x) + mask with x = scale q.k, c(x) = cap tanh(x / cap) under
// soft-capping (else x), and keys outside a query's 2-D neighbourhood or window
// are masked.  P = exp(s - LSE) uses the capped, masked score; the gradient
// with respect to x is dS c'(x), c'(x) = 1 - tanh^2(x / cap), and dQ, dK follow
// from x as above.  The additive mask has no gradient here.  Blocks that a 2-D
// mask hides entirely are computed (their P is 0), not skipped.
//
// Warps (320 threads): 0-7 elementwise (thread = TMEM lane = row; warps w and w + 4
// share a lane quarter and split each half block's columns), 8 TMA producer, 9 TMEM
// owner and MMA issuer (warp-uniform, elect.sync).  Every wait is bounded.
#pragma once

#include "fwd_common.cuh"

namespace attn_sm100 {

struct BwdParams {
    int B, Hq, Hkv, Nq, Nk, group;
    int nq_pad;          // row stride of the per-head D / LSE2 workspace (multiple of 128)
    float scale_log2;    // scale * log2(e)
    float scale;         // multiplies dQ and dK
    int is_causal;
    const int32_t* key_lens;
    const float* lse;    // forward LSE [B*Hq*Nq] (natural log)
    const uint16_t* o;   // forward O, bf16 [B*Hq*Nq*d]
    const uint16_t* dout;
    float* delta;        // workspace: D [B*Hq][nq_pad]
    float* lse2;         // workspace: LSE * log2(e); +inf for rows without keys and padding rows
    uint16_t* dq;        // bf16 [B*Hq*Nq*d]
    uint16_t* dk;        // bf16 [B*Hkv*Nk*d]
    uint16_t* dv;
    unsigned long long timeout_ns;
    unsigned int epoch;
    // variants (VAR instantiation): additive mask with element strides (b, h, q),
    // soft-capping (sc_in = 2 scale log2(e) / cap, sc_out = cap log2(e)), 2-D masks
    const float* mask;
    long long msb, msh, msq;
    int softcap_on;
    float sc_in, sc_out;
    int m2_kind, m2_w, m2_size, m2_shift;
    FastDiv fd_w, fd_size;
};

// Grid coordinates of token n under a 2-D mask, in the form the visibility test
// compares: (row, column) for a neighbourhood, the (row, column) window index for
// windows.
__device__ __forceinline__ int2 bwd_coord(const BwdParams& p, int n) {
    const int r = fdiv(n, p.fd_w);
    const int c = n - r * p.m2_w;
    if (p.m2_kind == 1) return make_int2(r, c);
    return make_int2(fdiv(r + p.m2_shift, p.fd_size), fdiv(c + p.m2_shift, p.fd_size));
}

__device__ __forceinline__ bool bwd_visible_2d(const BwdParams& p, int2 a, int2 b) {
    if (p.m2_kind == 1) return abs(a.x - b.x) < p.m2_size && abs(a.y - b.y) < p.m2_size;
    return a.x == b.x && a.y == b.y;
}

// Elementwise warps: kBwdSplit per TMEM lane quarter, each taking 1 / kBwdSplit of
// every half block's columns; then the TMA producer warp and the MMA warp.
constexpr int kBwdElemWarps = 8;
constexpr int kBwdSplit = kBwdElemWarps / 4;
constexpr int kBwdElemThreads = 32 * kBwdElemWarps;
constexpr int kBwdProducerWarp = kBwdElemWarps, kBwdMmaWarp = kBwdElemWarps + 1;
constexpr int kBwdThreads = 32 * (kBwdElemWarps + 2);
enum : unsigned int { kRoleBwdElem = 4, kRoleBwdProducer = 5, kRoleBwdMma = 6, kRoleBwdPrep = 7 };

// D_i = sum_t dO_it O_it and LSE2_i, one warp per (head, padded row).
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const BwdParams p) {
    const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const long long total = static_cast<long long>(p.B) * p.Hq * p.nq_pad;
    if (r >= total) return;
    const long long bh = r / p.nq_pad;
    const int i = static_cast<int>(r - bh * p.nq_pad);
    if (i >= p.Nq) {
        if (lane == 0) {
            p.delta[r] = 0.0f;
            p.lse2[r] = INFINITY;
        }
        return;
    }
    const long long row = bh * p.Nq + i;
    constexpr int kPer = D / 32;  // bf16 per lane
    const uint16_t* o = p.o + row * D + lane * kPer;
    const uint16_t* g = p.dout + row * D + lane * kPer;
    float acc = 0.0f;
    #pragma unroll
    for (int e = 0; e < kPer; e += 2) {
        const uint32_t ov = *reinterpret_cast<const uint32_t*>(o + e);
        const uint32_t gv = *reinterpret_cast<const uint32_t*>(g + e);
        acc = fmaf(__uint_as_float(ov << 16), __uint_as_float(gv << 16), acc);
        acc = fmaf(__uint_as_float(ov & 0xffff0000u), __uint_as_float(gv & 0xffff0000u), acc);
    }
    #pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) {
        const float l = p.lse[row];
        p.delta[r] = acc;
        p.lse2[r] = (l == -INFINITY) ? INFINITY : l * kLog2e;
    }
}

template <int D>
struct SmemBwd {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = 128 * 128;
    static constexpr int kTile = kChunks * kChunkBytes;  // 128 rows x D bf16, 128-byte swizzle
    // dK/dV kernel: K, V, then 2 stages of (Q, dO).  dQ kernel: Q, dO, then 2 stages of (K, V).
    static constexpr int kFixed0 = 0, kFixed1 = kTile;
    static constexpr int kStage = 2 * kTile;
    static constexpr int kStages = 2 * kTile;
    static constexpr int kBars = kStages + 2 * kStage;
    // barriers, per TMEM buffer b: STFULL + b (S and dP of a half block computed),
    // PFULL + b (P and dS of it stored); per stage s: RFULL + s, REMPTY + s
    static constexpr int FIXFULL = 0, DONE = 1, STFULL = 2, PFULL = 4, RFULL = 6, REMPTY = 8;
    static constexpr int FIXTM = 10;  // dQ kernel: Q and dO copied into TMEM (128 arrivals)
    static constexpr int kNumBars = 11;
    static constexpr int kMisc = kBars + 8 * kNumBars;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    // Two TMEM buffers of one half block (64 columns of the iteration's 128) each:
    // buffer b holds S (or S^T) in [128 b, 128 b + 64) and dP (dP^T) in
    // [128 b + 64, 128 b + 128); P and dS (bf16 pairs) of each 32-column chunk
    // overwrite the first 16 columns of that chunk.  The accumulators follow.
    static constexpr int kHalf = 64;
    static constexpr int kColBuf = 128, kColDP = 64, kColAcc0 = 256, kColAcc1 = 256 + D;
    // dQ kernel: the fixed Q and dO as bf16 pairs (D / 2 columns each), the A
    // operands of S and dP, so that only the streamed K and V come from shared memory
    static constexpr int kColFixT = 384;
    static_assert(kColFixT + D <= kTmemCols && kColAcc0 + D <= kColFixT, "TMEM budget of the dQ kernel");
    static_assert(kColAcc1 + D <= kTmemCols, "TMEM budget");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

// Writes one row of `D` fp32 TMEM columns, times `mul`, as bf16 to global `dst`
// (or zeros when `zero`), 32 columns per TMEM load.
template <int D>
__device__ __forceinline__ void store_row_bf16(uint32_t taddr, uint16_t* dst, float mul, bool zero, bool write,
                                               int c0 = 0, int nc = D / 32) {
    #pragma unroll
    for (int ci = 0; ci < D / 32; ++ci) {
        if (ci >= nc) break;
        const int c = c0 + ci;
        uint32_t v[32];
        if (!zero) {
            tmem_ld32(taddr + c * 32, v);
            tmem_wait_ld();
        }
        uint32_t w[16];
        #pragma unroll
        for (int e = 0; e < 16; ++e)
            w[e] = zero ? 0u : pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
        if (write) {
            uint4* out = reinterpret_cast<uint4*>(dst + c * 32);
            #pragma unroll
            for (int e = 0; e < 4; ++e) out[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
    }
}

// Shared structure of the two main kernels.  DKDV = true: rows of the TMEM
// tiles are keys, the fixed operands are K and V of one 128-key block, the
// streamed stages hold Q and dO of one query block.  DKDV = false: rows are
// queries, fixed Q and dO, streamed K and V.
template <int D, bool DKDV, bool VAR>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const BwdParams p) {
    using L = SmemBwd<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t sbase = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_base);
    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t limit = p.timeout_ns;

    // ---- the CTA's block and its loop
    const int blk = blockIdx.x;  // key block (DKDV) or query block
    int b, hk, h0;               // batch, K/V head, first query head
    int bh_fixed;                // z of the fixed operands' maps
    if constexpr (DKDV) {
        b = blockIdx.y / p.Hkv;
        hk = blockIdx.y - b * p.Hkv;
        h0 = hk * p.group;
        bh_fixed = blockIdx.y;  // b * Hkv + hk
    } else {
        b = blockIdx.y / p.Hq;
        h0 = blockIdx.y - b * p.Hq;
        hk = h0 / p.group;
        bh_fixed = blockIdx.y;  // b * Hq + h
    }
    int kv_len = p.key_lens != nullptr ? __ldg(p.key_lens + b) : p.Nk;
    if (kv_len < 0 || kv_len > p.Nk) {
        if (threadIdx.x == 0) record_error(kErrDevice, kRoleBwdElem, 1);
        kv_len = kv_len < 0 ? 0 : p.Nk;
    }
    const int n_qblk = (p.Nq + kBM - 1) / kBM;
    int n_iter, first;  // iterations: (query head, query block) pairs or key blocks
    if constexpr (DKDV) {
        first = p.is_causal ? blk : 0;  // query blocks that can see a key of this block
        const int per_head = blk * kBN < kv_len && first < n_qblk ? n_qblk - first : 0;
        n_iter = per_head * p.group;
    } else {
        int end = kv_len;
        if (p.is_causal && (blk + 1) * kBM < end) end = (blk + 1) * kBM;
        first = 0;
        n_iter = (end + kBN - 1) / kBN;
    }
    const int per_head = DKDV ? (n_qblk - first) : 1;
    auto iter_head = [&](int it) { return DKDV ? h0 + it / per_head : h0; };
    auto iter_blk = [&](int it) { return DKDV ? first + it % per_head : it; };

    if (threadIdx.x == 0) {
        mbar_init(bar(L::FIXFULL), 1);
        mbar_init(bar(L::DONE), 1);
        mbar_init(bar(L::FIXTM), kBwdElemThreads);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::STFULL + s), 1);
            mbar_init(bar(L::PFULL + s), kBwdElemThreads);
            mbar_init(bar(L::RFULL + s), 1);
            mbar_init(bar(L::REMPTY + s), 1);
        }
        *abort_flag = launch_aborted(p.epoch) ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == kBwdProducerWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kBwdProducerWarp) {
        // =============================== TMA producer ===============================
        if (lane == 0 && n_iter > 0 && !*abort_flag) {
            bool ok = true;
            int loads[2] = {0, 0};  // stage loads issued (RFULL phases)
            const uint32_t f0 = sbase + L::kFixed0, f1 = sbase + L::kFixed1;
            mbar_arrive_expect_tx(bar(L::FIXFULL), 2 * L::kTile);
            #pragma unroll
            for (int c = 0; c < L::kChunks; ++c) {
                if constexpr (DKDV) {
                    tma_load_3d(f0 + c * L::kChunkBytes, &tm_k, bar(L::FIXFULL), c * 64, blk * kBN, bh_fixed);
                    tma_load_3d(f1 + c * L::kChunkBytes, &tm_v, bar(L::FIXFULL), c * 64, blk * kBN, bh_fixed);
                } else {
                    tma_load_3d(f0 + c * L::kChunkBytes, &tm_q, bar(L::FIXFULL), c * 64, blk * kBM, bh_fixed);
                    tma_load_3d(f1 + c * L::kChunkBytes, &tm_do, bar(L::FIXFULL), c * 64, blk * kBM, bh_fixed);
                }
            }
            for (int it = 0; ok && it < n_iter; ++it) {
                const int s = it & 1;
                if (it >= 2 &&
                    !mbar_wait(bar(L::REMPTY + s), ((it >> 1) - 1) & 1, limit, abort_flag, p.epoch, kRoleBwdProducer, 1))
                    { ok = false; break; }
                const uint32_t st0 = sbase + L::kStages + s * L::kStage, st1 = st0 + L::kTile;
                const int ib = iter_blk(it);
                mbar_arrive_expect_tx(bar(L::RFULL + s), 2 * L::kTile);
                ++loads[s];
                #pragma unroll
                for (int c = 0; c < L::kChunks; ++c) {
                    if constexpr (DKDV) {
                        const int z = b * p.Hq + iter_head(it);
                        tma_load_3d(st0 + c * L::kChunkBytes, &tm_q, bar(L::RFULL + s), c * 64, ib * kBM, z);
                        tma_load_3d(st1 + c * L::kChunkBytes, &tm_do, bar(L::RFULL + s), c * 64, ib * kBM, z);
                    } else {
                        const int z = b * p.Hkv + hk;
                        tma_load_3d(st0 + c * L::kChunkBytes, &tm_k, bar(L::RFULL + s), c * 64, ib * kBN, z);
                        tma_load_3d(st1 + c * L::kChunkBytes, &tm_v, bar(L::RFULL + s), c * 64, ib * kBN, z);
                    }
                }
            }
            // every load issued has landed before the CTA may exit
            mbar_drain(bar(L::FIXFULL), 0, kRoleBwdProducer, 2);
            for (int s = 0; s < 2; ++s)
                if (loads[s] > 0) mbar_drain(bar(L::RFULL + s), (loads[s] - 1) & 1, kRoleBwdProducer, 3);
        }
    } else if (warp == kBwdMmaWarp) {
        // ================================ MMA issuer ================================
        // The iteration's 128 columns (queries for dK/dV, keys for dQ) go through the
        // tensor cores in two halves of 64, g = 2 it + hh, alternating between the two
        // TMEM buffers: while the elementwise warps turn S and dP of half g into P and
        // dS, the tensor cores run the accumulating products of half g - 1 and S, dP of
        // half g + 1.  Products of one thread run in order, so S of half g + 2 may
        // overwrite the buffer whose P and dS the products of half g read.
        constexpr uint32_t kIdescS = idesc_bf16_f32(128, L::kHalf, false);
        constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, true);
        bool ok = n_iter > 0 && !*abort_flag;
        if (ok) ok = mbar_wait_warp(bar(L::FIXFULL), 0, limit, abort_flag, p.epoch, kRoleBwdMma, 1);
        if (!DKDV && ok) ok = mbar_wait_warp(bar(L::FIXTM), 0, limit, abort_flag, p.epoch, kRoleBwdMma, 5);
        const uint32_t f0 = sbase + L::kFixed0, f1 = sbase + L::kFixed1;
        const int n_half = 2 * n_iter;
        // DKDV: S^T = K Q^T, dP^T = V dO^T.  dQ: S = Q K^T, dP = dO V^T.  A = fixed
        // (f0 / f1), B = the half's 64 rows of the streamed tiles (st0 / st1), K-major
        // over d; 64 rows are 8 KB into each 128-row, 128-byte swizzled chunk.
        auto issue_s = [&](int g) -> bool {
            const int it = g >> 1, hh = g & 1, s = it & 1, buf = g & 1;
            if (hh == 0 &&
                !mbar_wait_warp(bar(L::RFULL + s), (it >> 1) & 1, limit, abort_flag, p.epoch, kRoleBwdMma, 2))
                return false;
            tc_fence_after();
            const uint32_t st0 = sbase + L::kStages + s * L::kStage + hh * (L::kHalf * 128), st1 = st0 + L::kTile;
            const uint32_t cb = tmem + buf * L::kColBuf;
            // four K steps of 16 (32 bytes: +2 in descriptor units) per 64-column chunk,
            // issued by one elected lane per batch; the STFULL commit after the last
            #pragma unroll
            for (int f = 0; f < 2; ++f) {
                const uint32_t dst = cb + f * L::kColDP;
                const uint32_t bs = f == 0 ? st0 : st1;
                #pragma unroll
                for (int cc = 0; cc < L::kChunks; ++cc) {
                    const uint32_t commit = (f == 1 && cc == L::kChunks - 1) ? bar(L::STFULL + buf) : 0u;
                    const uint64_t bd = smem_desc_sw128(bs + cc * L::kChunkBytes, 16, 1024);
                    if constexpr (DKDV)
                        mma_ss_batch_warp<false, 4, 2, 2>(
                            dst, smem_desc_sw128((f == 0 ? f0 : f1) + cc * L::kChunkBytes, 16, 1024), bd, kIdescS,
                            cc > 0 ? 1u : 0u, commit);
                    else  // A = Q (or dO) from TMEM: 16 columns of d = 8 TMEM columns per step
                        mma_ts4_batch_warp<8, 2>(dst, tmem + L::kColFixT + f * (D / 2) + cc * 32, bd, kIdescS,
                                                 cc > 0 ? 1u : 0u, commit);
                }
            }
            return true;
        };
        for (int g = 0; ok && g < 2 && g < n_half; ++g) ok = issue_s(g);
        for (int g = 0; ok && g < n_half; ++g) {
            const int it = g >> 1, hh = g & 1, s = it & 1, buf = g & 1;
            if (!mbar_wait_warp(bar(L::PFULL + buf), (g >> 1) & 1, limit, abort_flag, p.epoch, kRoleBwdMma, 3))
                { ok = false; break; }
            tc_fence_after();
            // bf16 operands in TMEM (A) times the half's 64 streamed rows as B (MN-major,
            // 16 rows per step): DKDV: dV += P^T dO, dK += dS^T Q.  dQ: dQ += dS K.
            const uint32_t st0 = sbase + L::kStages + s * L::kStage, st1 = st0 + L::kTile;
            const uint32_t cb = tmem + buf * L::kColBuf;
            #pragma unroll
            for (int k4 = 0; k4 < L::kHalf / 16; ++k4) {
                const int kk = hh * (L::kHalf / 16) + k4;  // 16-row step within the 128 streamed rows
                // P and dS of 32-column chunk c sit in the first 16 columns of that chunk
                const uint32_t pc = (k4 >> 1) * 32 + (k4 & 1) * 8;
                const uint32_t acc = (g > 0 || k4 > 0) ? 1u : 0u;
                if constexpr (DKDV) {
                    mma_ts_warp(tmem + L::kColAcc0, cb + pc, smem_desc_sw128(st1 + kk * 2048, L::kChunkBytes, 1024),
                                kIdescAcc, acc);
                    mma_ts_warp(tmem + L::kColAcc1, cb + L::kColDP + pc,
                                smem_desc_sw128(st0 + kk * 2048, L::kChunkBytes, 1024), kIdescAcc, acc);
                } else {
                    mma_ts_warp(tmem + L::kColAcc0, cb + L::kColDP + pc,
                                smem_desc_sw128(st0 + kk * 2048, L::kChunkBytes, 1024), kIdescAcc, acc);
                }
            }
            if (hh == 1) mma_commit_warp(bar(L::REMPTY + s));  // the stage may be refilled once these complete
            if (g + 2 < n_half && !issue_s(g + 2)) { ok = false; break; }
        }
        mma_commit_warp(bar(L::DONE));
        mbar_drain(bar(L::DONE), 0, kRoleBwdMma, 4);
    } else {
        // ============================ elementwise warps =============================
        const int quarter = warp & 3, sub = warp >> 2;  // TMEM lane quarter, column share
        const int row = quarter * 32 + lane;            // TMEM lane
        const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const float c2 = p.scale_log2;
        // per-row constants of the dQ kernel (rows are queries)
        const int q_row = DKDV ? 0 : blk * kBM + row;
        float my_lse2 = 0.0f, my_d = 0.0f;
        if constexpr (!DKDV) {
            const long long r = static_cast<long long>(blockIdx.y) * p.nq_pad + q_row;
            my_lse2 = p.lse2[r];
            my_d = p.delta[r];
        }
        const int key_row = DKDV ? blk * kBN + row : 0;
        // DKDV: LSE2 and D of each iteration's 128 queries, one value per thread of the
        // first warp of each lane quarter, stored at the start of the iteration from
        // registers loaded one iteration earlier, and shared through a double buffer (a
        // buffer is rewritten two iterations later, after every thread has passed the
        // barrier of the iteration between)
        __shared__ __align__(16) float s_l2[2][kBM];
        __shared__ __align__(16) float s_dd[2][kBM];
        // VAR with a 2-D mask: grid coordinates of this iteration's columns (queries
        // or keys), double-buffered like LSE2 and D, and of this thread's own row
        __shared__ int2 s_xy[2][kBM];
        const bool m2 = VAR && p.m2_kind != 0;
        int2 my_xy = make_int2(0, 0);
        if (m2) my_xy = bwd_coord(p, DKDV ? key_row : q_row);
        bool ok = !*abort_flag;
        if constexpr (!DKDV) {
            // Q and dO of this CTA's 128 rows into TMEM (this thread's row: lane = row,
            // bf16 pairs along d), read from their 128-byte swizzled shared-memory tiles
            if (n_iter > 0) {
                if (ok) {
                    const bool got = mbar_wait(bar(L::FIXFULL), 0, limit, abort_flag, p.epoch, kRoleBwdElem, 4);
                    ok = __all_sync(0xffffffffu, got);
                }
                if (ok) {
                    #pragma unroll
                    for (int f = 0; f < 2; ++f) {
                        if (kBwdSplit == 2 && f != sub) continue;  // Q by one warp of the quarter, dO by the other
                        const uint8_t* tile = smem + (f == 0 ? L::kFixed0 : L::kFixed1);
                        #pragma unroll
                        for (int c = 0; c < L::kChunks; ++c) {
                            uint32_t w[32];
                            #pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const uint4 v = *reinterpret_cast<const uint4*>(
                                    tile + c * L::kChunkBytes + row * 128 + ((u ^ (row & 7)) << 4));
                                w[4 * u] = v.x; w[4 * u + 1] = v.y; w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
                            }
                            tmem_st32(lane_tmem + L::kColFixT + f * (D / 2) + c * 32, w);
                        }
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                mbar_arrive(bar(L::FIXTM));  // also after a failed wait: the MMA warp then finds the abort
            }
        }
        // DKDV: LSE2 and D of query `row` of an iteration's block, loaded one iteration
        // ahead into registers so that their latency overlaps the previous iteration
        // (rows are padded to a multiple of 128 per head: row < 128 stays in bounds)
        float pre_l2 = 0.0f, pre_dd = 0.0f;
        auto prefetch_rows = [&](int it2) {
            if (DKDV && sub == 0 && it2 < n_iter) {
                const long long r = static_cast<long long>(b * p.Hq + iter_head(it2)) * p.nq_pad + iter_blk(it2) * kBM;
                pre_l2 = __ldg(p.lse2 + r + row);
                pre_dd = __ldg(p.delta + r + row);
            }
        };
        prefetch_rows(0);
        // Every warp runs the named barrier of every iteration, also after a failed
        // wait (it then skips the iteration's work), so that none is left waiting.
        for (int it = 0; it < n_iter; ++it) {
            const int ib = iter_blk(it);
            // DKDV: LSE2 and D of this iteration's 128 queries in shared memory, read by
            // every lane at the same address (broadcast loads)
            const int buf = it & 1;
            if constexpr (DKDV) {
                if (sub == 0) {
                    s_l2[buf][row] = pre_l2;
                    s_dd[buf][row] = pre_dd;
                    if (m2) s_xy[buf][row] = bwd_coord(p, ib * kBM + row);
                }
                named_barrier_sync(1, kBwdElemThreads);
                prefetch_rows(it + 1);
            } else if (m2) {
                if (sub == 0) s_xy[buf][row] = bwd_coord(p, ib * kBN + row);
                named_barrier_sync(1, kBwdElemThreads);
            }
            // VAR: the additive mask row of this thread (DKDV: column = query, row = key)
            const float* mrow = nullptr;
            if (VAR && p.mask != nullptr) {
                if constexpr (DKDV)
                    mrow = p.mask + static_cast<long long>(b) * p.msb + static_cast<long long>(iter_head(it)) * p.msh +
                           static_cast<long long>(ib) * kBM * p.msq + key_row;
                else
                    mrow = p.mask + static_cast<long long>(b) * p.msb + static_cast<long long>(h0) * p.msh +
                           static_cast<long long>(q_row) * p.msq + static_cast<long long>(ib) * kBN;
            }
            if (!ok) continue;
            for (int hh = 0; hh < 2 && ok; ++hh) {
                const int g = 2 * it + hh, hb = g & 1;
                const bool got = mbar_wait(bar(L::STFULL + hb), (g >> 1) & 1, limit, abort_flag, p.epoch,
                                           kRoleBwdElem, 2);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                const uint32_t cb = lane_tmem + hb * L::kColBuf;
                // Every score of the half visible for every row of the warp (no key past
                // the key length, no pair across the causal diagonal): no per-element test.
                bool all_vis;
                if constexpr (DKDV) {
                    const int q_first = ib * kBM + hh * L::kHalf;
                    all_vis = key_row < kv_len && (!p.is_causal || key_row <= q_first);
                } else {
                    const int k_last = ib * kBN + hh * L::kHalf + L::kHalf - 1;
                    all_vis = k_last < kv_len && (!p.is_causal || k_last <= q_row);
                }
                all_vis = __all_sync(0xffffffffu, all_vis);
                constexpr int kMyChunks = L::kHalf / 32 / kBwdSplit;  // 32-column chunks of this warp
                if (!VAR && all_vis) {
                    #pragma unroll
                    for (int ci = 0; ci < kMyChunks; ++ci) {
                        const int c = sub * kMyChunks + ci;
                        uint32_t sv[32], dv[32];
                        tmem_ld32(cb + c * 32, sv);
                        tmem_ld32(cb + L::kColDP + c * 32, dv);
                        tmem_wait_ld();
                        uint32_t pw[16], dw[16];
                        #pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            float l2[4], dd[4];
                            if constexpr (DKDV) {
                                // the same 16 bytes in every lane: broadcast loads
                                const int col = hh * L::kHalf + c * 32 + e;
                                const float4 a = *reinterpret_cast<const float4*>(&s_l2[buf][col]);
                                const float4 b4 = *reinterpret_cast<const float4*>(&s_dd[buf][col]);
                                l2[0] = a.x; l2[1] = a.y; l2[2] = a.z; l2[3] = a.w;
                                dd[0] = b4.x; dd[1] = b4.y; dd[2] = b4.z; dd[3] = b4.w;
                            } else {
                                #pragma unroll
                                for (int u = 0; u < 4; ++u) { l2[u] = my_lse2; dd[u] = my_d; }
                            }
                            float pv[4], ds[4];
                            #pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                pv[u] = ex2_approx(fmaf(__uint_as_float(sv[e + u]), c2, -l2[u]));
                                ds[u] = pv[u] * (__uint_as_float(dv[e + u]) - dd[u]);
                            }
                            pw[e / 2] = pack_bf16x2(pv[0], pv[1]);
                            pw[e / 2 + 1] = pack_bf16x2(pv[2], pv[3]);
                            dw[e / 2] = pack_bf16x2(ds[0], ds[1]);
                            dw[e / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
                        }
                        if constexpr (DKDV) tmem_st16(cb + c * 32, pw);
                        tmem_st16(cb + L::kColDP + c * 32, dw);
                    }
                } else {
                #pragma unroll
                for (int ci = 0; ci < kMyChunks; ++ci) {
                    const int c = sub * kMyChunks + ci;
                    uint32_t sv[32], dv[32];
                    tmem_ld32(cb + c * 32, sv);
                    tmem_ld32(cb + L::kColDP + c * 32, dv);
                    tmem_wait_ld();
                    uint32_t pw[16], dw[16];
                    #pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float pp[2], ds[2];
                        #pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            // query (DKDV) or key (dQ) within the iteration's 128
                            const int col = hh * L::kHalf + c * 32 + e + u;
                            float l2, dd;
                            bool vis;
                            if constexpr (DKDV) {
                                const int qi = ib * kBM + col;
                                l2 = s_l2[buf][col];  // the same address in every lane: a broadcast
                                dd = s_dd[buf][col];
                                vis = key_row < kv_len && (!p.is_causal || key_row <= qi);
                            } else {
                                const int kj = ib * kBN + col;
                                l2 = my_lse2;
                                dd = my_d;
                                vis = kj < kv_len && (!p.is_causal || kj <= q_row);
                            }
                            if constexpr (!VAR) {
                                const float pv = vis ? ex2_approx(fmaf(__uint_as_float(sv[e + u]), c2, -l2)) : 0.0f;
                                pp[u] = pv;
                                ds[u] = pv * (__uint_as_float(dv[e + u]) - dd);
                            } else {
                                // base-2 logit of the capped, masked score, and c'(x)
                                const float raw = __uint_as_float(sv[e + u]);
                                float lg = raw * c2, gd = 1.0f;
                                if (p.softcap_on) {
                                    const float t = fmaf(rcp_approx(1.0f + ex2_approx(raw * p.sc_in)), -2.0f, 1.0f);
                                    lg = p.sc_out * t;
                                    gd = fmaf(-t, t, 1.0f);
                                }
                                if (m2) vis = vis && bwd_visible_2d(p, my_xy, s_xy[buf][col]);
                                // (padding query rows past Nq have no mask row: not read)
                                if (mrow != nullptr && vis && (DKDV ? ib * kBM + col < p.Nq : q_row < p.Nq)) {
                                    const long long off = DKDV ? static_cast<long long>(col) * p.msq : col;
                                    lg = fmaf(__ldg(mrow + off), kLog2e, lg);
                                }
                                const float pv = vis ? ex2_approx(lg - l2) : 0.0f;
                                pp[u] = pv;
                                ds[u] = pv * (__uint_as_float(dv[e + u]) - dd) * gd;
                            }
                        }
                        pw[e / 2] = pack_bf16x2(pp[0], pp[1]);
                        dw[e / 2] = pack_bf16x2(ds[0], ds[1]);
                    }
                    // P (DKDV only) over this chunk's S columns, already read by this
                    // thread, dS over its dP columns (a warp sharing the lane quarter
                    // reads the other chunk: no store may land there)
                    if constexpr (DKDV) tmem_st16(cb + c * 32, pw);
                    tmem_st16(cb + L::kColDP + c * 32, dw);
                }
                }
                // the half's P and dS stored: its products may start
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(L::PFULL + hb));
            }
        }
        // ------------------------------------------------------------- epilogue
        bool have = n_iter > 0 && ok;
        if (have) {
            const bool got = mbar_wait(bar(L::DONE), 0, limit, abort_flag, p.epoch, kRoleBwdElem, 3);
            have = __all_sync(0xffffffffu, got);
            tc_fence_after();
        }
        const bool failed = n_iter > 0 && !have;
        if (!failed) {
            if constexpr (DKDV) {
                const bool write = key_row < p.Nk;
                const long long base = (static_cast<long long>(b * p.Hkv + hk) * p.Nk + key_row) * D;
                if (kBwdSplit == 1 || sub == 0)
                    store_row_bf16<D>(lane_tmem + L::kColAcc0, p.dv + base, 1.0f, n_iter == 0, write);
                if (kBwdSplit == 1 || sub == 1)
                    store_row_bf16<D>(lane_tmem + L::kColAcc1, p.dk + base, p.scale, n_iter == 0, write);
            } else {
                const bool write = q_row < p.Nq;
                const long long base = (static_cast<long long>(blockIdx.y) * p.Nq + q_row) * D;
                constexpr int kMine = D / 32 / kBwdSplit;  // 32-column chunks of dQ this warp writes
                store_row_bf16<D>(lane_tmem + L::kColAcc0, p.dq + base, p.scale, n_iter == 0, write, sub * kMine,
                                  kMine);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn_sm100
