// decode_kernel.cuh -- split-KV attention for decoding-shaped inputs (few query
// rows per head, long key sequences) on sm_100a.
//
// The decoding phase of "FlashAttention technical analysis"
// (jsqmd.com/news/722897), section 5.2, needs FlashDecoding: the keys of each
// head are cut into ranges processed in parallel and merged by their
// log-sum-exp.  With R = (query heads per K/V head) x Nq <= 16 rows per K/V
// head, the work is a skinny matrix product per K/V head and the kernel is
// bound by HBM bandwidth: every K/V byte is read once and used by all R rows.
//
//   one CTA per (batch, K/V head, key range); all R query rows of the group
//   share every K/V row, which is read from HBM once (TMA, 32-key chunks with
//   128-byte swizzle); the consumer warps take the chunks round-robin, each
//   through its own ring of shared-memory stages (so that a warp never waits on
//   a stage another warp may still hold).  A warp computes S = Q K^T of its
//   chunk and O += P V with warp-level bf16 tensor-core tiles (m16n8k16, the
//   R rows padded to 16, fp32 accumulation; ldmatrix from the swizzled stages),
//   with the online softmax on the S fragments in fp32; its running max, sum
//   and output stay in registers.  The warps merge in shared memory and the
//   CTA writes its range's normalised O and LSE to the split-KV workspace,
//   merged by attn_splitkv_combine_kernel.  The instruction count per chunk
//   does not depend on R, so every R <= 16 streams K/V at the same rate.
//
// Masks: key lengths only (no causal mask, no additive mask).
#pragma once

#include "fwd_common.cuh"

namespace attn_sm100 {

constexpr int kDecWarps = 6;                       // consumer warps
constexpr int kDecThreads = (kDecWarps + 1) * 32;  // + 1 TMA producer warp
constexpr int kDecChunk = 32;                      // keys per chunk (one per lane)
constexpr int kDecMaxRows = 16;

struct DecParams {
    int B, Hq, Hkv, Nq, Nk, group, rows;  // rows = group * Nq
    float scale_log2;
    const int32_t* key_lens;
    const uint16_t* q;  // bf16 [B, Hq, Nq, d]
    int n_splits, split_keys;  // split_keys: a multiple of kDecChunk
    float* ws_o;    // [n_splits][B * Hq * Nq][d]
    float* ws_lse;  // [n_splits][B * Hq * Nq]
    unsigned long long timeout_ns;
    unsigned int epoch;
};

template <int D>
struct SmemDec {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = kDecChunk * 128;         // 32 rows x 64 bf16, 128-byte swizzle
    static constexpr int kTensorBytes = kHalves * kHalfBytes;  // K (or V) of one chunk
    static constexpr int kStageBytes = 2 * kTensorBytes;
    static constexpr int kPerWarp = D == 128 ? 2 : 4;          // stages of each consumer warp
    static constexpr int kStages = kDecWarps * kPerWarp;
    static constexpr int kQ = kStages * kStageBytes;           // bf16 [kDecMaxRows][D], rows >= R zero
    // per-warp results for the merge, after the last chunk (over the stage ring):
    // m [rows], l [rows], O [rows][D]
    static constexpr int kMergeWarp = 2 * kDecMaxRows * 4 + kDecMaxRows * D * 4;
    static constexpr int kBars = kQ + kDecMaxRows * D * 2;
    static constexpr int kNumBars = 2 * kStages;
    static constexpr int kMisc = kBars + 8 * kNumBars;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kDecWarps * kMergeWarp <= kQ, "merge area inside the stage ring");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

// Byte offset of element (row j, column t) of a chunk tile: 64-column halves of
// 32 rows x 128 bytes, 16-byte units permuted by (row & 7) (the TMA 128-byte swizzle).
__device__ __forceinline__ uint32_t dec_swz(int j, int t) {
    return (t >> 6) * SmemDec<64>::kHalfBytes + j * 128 + ((((t & 63) >> 3) ^ (j & 7)) << 4) + ((t & 7) << 1);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const DecParams p) {
    using L = SmemDec<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t sbase = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_base);
    auto full = [&](int s) -> uint32_t { return sbase + L::kBars + 8u * s; };
    auto empty = [&](int s) -> uint32_t { return sbase + L::kBars + 8u * (L::kStages + s); };
    // chunk c: consumer warp c % kDecWarps, its (c / kDecWarps)-th chunk, in that warp's own stages
    auto stage_of = [&](int c) { return (c % kDecWarps) * L::kPerWarp + (c / kDecWarps) % L::kPerWarp; };
    auto use_of = [&](int c) { return (c / kDecWarps) / L::kPerWarp; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t limit = p.timeout_ns;
    // CTA -> (batch, K/V head, key range)
    const int split = blockIdx.x % p.n_splits;
    const int bhk = blockIdx.x / p.n_splits;
    const int b = bhk / p.Hkv, hk = bhk - (bhk / p.Hkv) * p.Hkv;
    int kv_len = p.key_lens != nullptr ? __ldg(p.key_lens + b) : p.Nk;
    if (kv_len < 0 || kv_len > p.Nk) {
        if (threadIdx.x == 0) record_error(kErrDevice, kRoleSoftmax, 2);
        kv_len = kv_len < 0 ? 0 : p.Nk;
    }
    const int k_lo = split * p.split_keys;
    const int k_hi = (k_lo + p.split_keys < kv_len) ? k_lo + p.split_keys : kv_len;
    const int n_chunks = k_hi > k_lo ? (k_hi - k_lo + kDecChunk - 1) / kDecChunk : 0;
    const int R = p.rows;

    uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L::kQ);
    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        *abort_flag = launch_aborted(p.epoch) ? 1 : 0;
        fence_mbar_init();
    }
    // Q of the group's R rows (bf16 as given; row r = g * Nq + i), rows R..15 zero
    for (int e = threadIdx.x; e < kDecMaxRows * D; e += kDecThreads) {
        const int r = e / D, t = e - r * D;
        uint16_t val = 0;
        if (r < R) {
            const int g = r / p.Nq, i = r - g * p.Nq;
            val = p.q[((static_cast<long long>(b) * p.Hq + hk * p.group + g) * p.Nq + i) * D + t];
        }
        qs[e] = val;
    }
    __syncthreads();

    if (warp == kDecWarps) {
        // =============================== TMA producer ===============================
        if (lane == 0 && !*abort_flag) {
            int issued = 0;
            for (int c = 0; c < n_chunks; ++c) {
                const int s = stage_of(c), u = use_of(c);
                if (u > 0 && !mbar_wait(empty(s), (u - 1) & 1, limit, abort_flag, p.epoch, kRoleProducer, 40))
                    break;
                const uint32_t dst = sbase + s * L::kStageBytes;
                mbar_arrive_expect_tx(full(s), L::kStageBytes);
                #pragma unroll
                for (int h = 0; h < L::kHalves; ++h) {
                    tma_load_3d(dst + h * L::kHalfBytes, &tm_k, full(s), h * 64, k_lo + c * kDecChunk, bhk);
                    tma_load_3d(dst + L::kTensorBytes + h * L::kHalfBytes, &tm_v, full(s), h * 64,
                                k_lo + c * kDecChunk, bhk);
                }
                issued = c + 1;
            }
            // every load issued has landed: the last use of each stage
            for (int c = issued - 1; c >= 0 && c >= issued - L::kStages; --c)
                mbar_drain(full(stage_of(c)), use_of(c) & 1, kRoleProducer, 41);
        }
    } else {
        // ============================== consumer warps ==============================
        // Fragments of m16n8k16: lane = 4 * row-in-8 + quad position; a lane holds
        // rows r0 = lane / 4 and r1 = r0 + 8, columns 2 * (lane % 4) + {0, 1} of
        // every 8-column tile.
        const int r0 = lane >> 2, qc = 2 * (lane & 3);
        // Q as A fragments, one per 16 columns of d (ldmatrix: lane -> row lane % 16,
        // columns 8 * (lane / 16) of the 16-column slice)
        uint32_t qa[D / 16][4];
        #pragma unroll
        for (int kt = 0; kt < D / 16; ++kt)
            ldsm_x4(smem_u32(qs + (lane & 15) * D + kt * 16 + (lane >> 4) * 8), qa[kt]);
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
        float o[D / 8][4];
        #pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
        const float c2 = p.scale_log2;
        bool ok = true;
        for (int c = warp; ok && c < n_chunks; c += kDecWarps) {
            const int s = stage_of(c);
            const bool got = mbar_wait(full(s), use_of(c) & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 42);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            const uint32_t kt_s = sbase + s * L::kStageBytes;
            const uint32_t vt_s = kt_s + L::kTensorBytes;
            // ---- S = Q K^T: 4 tiles of 8 keys.  ldmatrix (no transpose) of K rows gives
            // the column-major B fragment; one x4 load covers two 16-column k steps.
            float sc[4][4];
            #pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
                #pragma unroll
                for (int kt = 0; kt < D / 16; kt += 2) {
                    // matrix lane / 8: k step kt + (lane / 16), half (lane / 8) % 2
                    const int key = nt * 8 + (lane & 7);
                    const int col = (kt + (lane >> 4)) * 16 + ((lane >> 3) & 1) * 8;
                    uint32_t bk[4];
                    ldsm_x4(kt_s + dec_swz(key, col), bk);
                    mma_bf16_16816(sc[nt], qa[kt], bk[0], bk[1]);
                    mma_bf16_16816(sc[nt], qa[kt + 1], bk[2], bk[3]);
                }
            }
            // ---- online softmax on the fragments (base 2, lazy rescale 2^8)
            const int key0 = k_lo + c * kDecChunk;
            #pragma unroll
            for (int h = 0; h < 2; ++h) {  // h = 0: row r0, h = 1: row r1
                float mx = -INFINITY;
                #pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int key = key0 + nt * 8 + qc + e;
                        const float v = key < k_hi ? sc[nt][2 * h + e] * c2 : -INFINITY;
                        sc[nt][2 * h + e] = v;
                        mx = fmaxf(mx, v);
                    }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                if (mx > m[h] + kLazyTau) {  // the same decision in the 4 lanes of the row
                    const float alpha = (m[h] == -INFINITY) ? 0.0f : ex2_approx(m[h] - mx);
                    l[h] *= alpha;
                    #pragma unroll
                    for (int nt = 0; nt < D / 8; ++nt) {
                        o[nt][2 * h] *= alpha;
                        o[nt][2 * h + 1] *= alpha;
                    }
                    m[h] = mx;
                }
                #pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float pv = (m[h] == -INFINITY) ? 0.0f : ex2_approx(sc[nt][2 * h + e] - m[h]);
                        sc[nt][2 * h + e] = pv;
                        l[h] += pv;  // this lane's share of the row sum
                    }
            }
            // ---- O += P V: P's C fragments of two 8-key tiles are the A fragment of one
            // 16-key step; V through ldmatrix.trans (rows = keys) is the B fragment.
            #pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                uint32_t pa[4];
                pa[0] = pack_bf16x2(sc[2 * k2][0], sc[2 * k2][1]);
                pa[1] = pack_bf16x2(sc[2 * k2][2], sc[2 * k2][3]);
                pa[2] = pack_bf16x2(sc[2 * k2 + 1][0], sc[2 * k2 + 1][1]);
                pa[3] = pack_bf16x2(sc[2 * k2 + 1][2], sc[2 * k2 + 1][3]);
                #pragma unroll
                for (int nt = 0; nt < D / 8; nt += 2) {
                    // matrix lane / 8: keys 16 k2 + 8 * ((lane / 8) % 2), columns 8 * (nt + lane / 16)
                    const int key = k2 * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                    const int col = (nt + (lane >> 4)) * 8;
                    uint32_t bv[4];
                    ldsm_x4_t(vt_s + dec_swz(key, col), bv);
                    mma_bf16_16816(o[nt], pa, bv[0], bv[1]);
                    mma_bf16_16816(o[nt + 1], pa, bv[2], bv[3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(s));  // this warp has read the chunk
        }
        // ---- per-warp results to shared memory (over the stage ring, once every
        // warp is done with it and every load has landed)
        named_barrier_sync(1, kDecWarps * 32);
        float* mw = reinterpret_cast<float*>(smem + warp * L::kMergeWarp);
        float* lw = mw + kDecMaxRows;
        float* ow = lw + kDecMaxRows;
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = r0 + 8 * h;
            float lr = l[h];
            lr += __shfl_xor_sync(0xffffffffu, lr, 1);
            lr += __shfl_xor_sync(0xffffffffu, lr, 2);
            if ((lane & 3) == 0) {
                mw[r] = ok ? m[h] : -INFINITY;
                lw[r] = ok ? lr : 0.0f;
            }
            #pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                ow[r * D + nt * 8 + qc] = ok ? o[nt][2 * h] : 0.0f;
                ow[r * D + nt * 8 + qc + 1] = ok ? o[nt][2 * h + 1] : 0.0f;
            }
        }
    }
    __syncthreads();
    // ---- merge the warps and write this range's result: thread = (row, column)
    if (!*abort_flag) {
        for (int e = threadIdx.x; e < R * D; e += kDecThreads) {
            const int r = e / D, t = e - r * D;
            float M = -INFINITY;
            #pragma unroll
            for (int w = 0; w < kDecWarps; ++w)
                M = fmaxf(M, reinterpret_cast<const float*>(smem + w * L::kMergeWarp)[r]);
            float lsum = 0.0f, osum = 0.0f;
            if (M != -INFINITY) {
                #pragma unroll
                for (int w = 0; w < kDecWarps; ++w) {
                    const float* mw = reinterpret_cast<const float*>(smem + w * L::kMergeWarp);
                    const float a = (mw[r] == -INFINITY) ? 0.0f : ex2_approx(mw[r] - M);
                    lsum = fmaf(a, mw[kDecMaxRows + r], lsum);
                    osum = fmaf(a, mw[2 * kDecMaxRows + r * D + t], osum);
                }
            }
            const int g = r / p.Nq, i = r - g * p.Nq;
            const long long row = (static_cast<long long>(b) * p.Hq + hk * p.group + g) * p.Nq + i;
            const long long rs = static_cast<long long>(split) * p.B * p.Hq * p.Nq + row;
            p.ws_o[rs * D + t] = lsum > 0.0f ? osum / lsum : 0.0f;
            if (t == 0) p.ws_lse[rs] = lsum > 0.0f ? (M + __log2f(lsum)) * kLn2 : -INFINITY;
        }
    }
}

}  // namespace attn_sm100
