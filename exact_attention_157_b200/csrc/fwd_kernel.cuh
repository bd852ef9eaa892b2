// fwd_kernel.cuh -- exact attention forward pass for sm_100a.
//
// One CTA computes one 128-row query tile of one (batch, query head):
//
//   warp 4      TMA producer: Q tile once, then K_j / V_j key blocks into two
//               NS-stage shared-memory rings (128-byte swizzle, no multicast).
//   warp 5      tensor-memory owner and MMA issuer (one thread):
//                 S_j  = Q K_j^T     tcgen05.mma, A and B from shared memory,
//                                     fp32 accumulator in TMEM, double-buffered;
//                 O   += P_j V_j     tcgen05.mma, A = P_j from TMEM (bf16),
//                                     B = V_j from shared memory (N-major).
//               Issue order S_0, S_1, PV_0, S_2, PV_1, ... so that the tensor
//               cores work on S_{j+1} and PV_{j-1} while the softmax warps
//               process S_j.
//   warps 0-3   softmax, one thread per query row (TMEM lane): online softmax
//               with a running max m and running sum l ("FlashAttention
//               technical analysis", jsqmd.com/news/722897, section 2.2) in the
//               base-2 domain with the scale folded into one FMA; the output
//               correction is lazy (only when the max grows by more than
//               2^8, the deferred rescaling of section 4.1 taken further);
//               one final normalisation O / l, the per-row LSE, and the
//               epilogue through shared memory and a TMA store.
//
// Masks are applied per element only on blocks that cross a key-length or
// causal boundary; blocks past the boundary are never loaded or multiplied.
// Every wait is bounded (see sm100_ptx.cuh); on expiry the roles stop, drain
// what they issued, and the CTA frees its tensor memory and returns.
#pragma once

#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int kBM = 128;          // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;          // keys per block
constexpr int kThreads = 192;     // 6 warps
constexpr int kTmemCols = 512;
constexpr float kLazyTau = 8.0f;  // rescale only when the max grows by > 2^8
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Roles for error reporting.
enum : unsigned int { kRoleSoftmax = 1, kRoleProducer = 2, kRoleMma = 3, kRoleSelftest = 9 };

struct FwdParams {
    int B, Hq, Hkv, Nq, Nk;
    int group;          // Hq / Hkv
    int n_qtiles;       // ceil(Nq / 128)
    float scale_log2;   // softmax scale * log2(e), > 0
    int is_causal;
    const int32_t* key_lens;
    const float* mask;
    long long msb, msh, msq;
    float* lse;
    void* out;     // O base (bf16), for rows written without the TMA store
    int unit_run;  // persistent kernel: consecutive units per CTA turn (1 or 2)
    unsigned long long timeout_ns;
    unsigned int epoch;  // launch id for the launch-wide abort (never 0)
};

template <int D, int NS>
struct Smem {
    static constexpr int kChunks = D / 64;               // 128-byte-wide column chunks
    static constexpr int kChunkBytes = 128 * 128;        // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kQ = 0;
    static constexpr int kK = kTileBytes;
    static constexpr int kV = kK + NS * kTileBytes;
    static constexpr int kBars = kV + NS * kTileBytes;
    // barrier indices
    static constexpr int QFULL = 0;
    static constexpr int KFULL = 1;
    static constexpr int KEMPTY = 1 + NS;
    static constexpr int VFULL = 1 + 2 * NS;
    static constexpr int VEMPTY = 1 + 3 * NS;
    static constexpr int SFULL = 1 + 4 * NS;   // 2
    static constexpr int PFULL = 3 + 4 * NS;   // 2
    static constexpr int ODONE = 5 + 4 * NS;   // one phase per PV (used only while PV_{j-2} is known done)
    static constexpr int OFINAL = 6 + 4 * NS;  // the last PV only: the epilogue's wait
    static constexpr int MMAFIN = 7 + 4 * NS;
    static constexpr int kNumBars = 8 + 4 * NS;
    static constexpr int kMisc = kBars + 8 * kNumBars;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
    // TMEM column map
    static constexpr int kColS = 0;                // S_0 at 0, S_1 at 128
    static constexpr int kColO = 256;
    static constexpr int kColP = 256 + D;          // P_0, P_1: 64 columns each (bf16 pairs)
    static_assert(kColP + 128 <= kTmemCols, "TMEM budget");
};

template <int D, int NS, bool HAS_MASK>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const FwdParams p) {
    using L = Smem<D, NS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t sbase = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- tile coordinates (heavier causal tiles of a head start first)
    const int bh = blockIdx.x / p.n_qtiles;
    int qt = blockIdx.x % p.n_qtiles;
    if (p.is_causal) qt = p.n_qtiles - 1 - qt;
    const int b = bh / p.Hq;
    const int h = bh - b * p.Hq;
    const int bhk = b * p.Hkv + h / p.group;
    const int q0 = qt * kBM;
    int kv_len = p.Nk;
    if (p.key_lens != nullptr) {
        kv_len = p.key_lens[b];
        if (kv_len < 0 || kv_len > p.Nk) {
            if (threadIdx.x == 0) record_error(kErrDevice, kRoleSoftmax, 1);
            kv_len = kv_len < 0 ? 0 : p.Nk;
        }
    }
    int kv_end = kv_len;
    if (p.is_causal && q0 + kBM < kv_end) kv_end = q0 + kBM;
    int n_blocks = (kv_end + kBN - 1) / kBN;

    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(L::QFULL), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(L::KFULL + s), 1);
            mbar_init(bar(L::KEMPTY + s), 1);
            mbar_init(bar(L::VFULL + s), 1);
            mbar_init(bar(L::VEMPTY + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(L::SFULL + i), 1);
            mbar_init(bar(L::PFULL + i), 128);
        }
        mbar_init(bar(L::ODONE), 1);
        mbar_init(bar(L::OFINAL), 1);
        mbar_init(bar(L::MMAFIN), 1);
        // A CTA that starts after another CTA of this launch timed out does no work.
        *abort_flag = launch_aborted(p.epoch) ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
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
    if (*abort_flag) n_blocks = 0;
    n_blocks = __shfl_sync(0xffffffffu, n_blocks, 0);  // warp-uniform from here on

    if (warp == 4) {
        // ============================== TMA producer ==============================
        if (lane == 0 && n_blocks > 0) {
            int k_uses[NS], v_uses[NS];
            #pragma unroll
            for (int s = 0; s < NS; ++s) { k_uses[s] = 0; v_uses[s] = 0; }
            mbar_arrive_expect_tx(bar(L::QFULL), L::kTileBytes);
            #pragma unroll
            for (int c = 0; c < L::kChunks; ++c)
                tma_load_3d(sbase + L::kQ + c * L::kChunkBytes, &tm_q, bar(L::QFULL), c * 64, q0, bh);
            for (int j = 0; j < n_blocks; ++j) {
                const int s = j % NS;
                const int use = j / NS;
                if (use > 0 && !mbar_wait(bar(L::KEMPTY + s), (use - 1) & 1, limit, abort_flag, p.epoch, kRoleProducer, 10))
                    break;
                mbar_arrive_expect_tx(bar(L::KFULL + s), L::kTileBytes);
                #pragma unroll
                for (int c = 0; c < L::kChunks; ++c)
                    tma_load_3d(sbase + L::kK + s * L::kTileBytes + c * L::kChunkBytes, &tm_k,
                                bar(L::KFULL + s), c * 64, j * kBN, bhk);
                k_uses[s] = use + 1;
                if (use > 0 && !mbar_wait(bar(L::VEMPTY + s), (use - 1) & 1, limit, abort_flag, p.epoch, kRoleProducer, 11))
                    break;
                mbar_arrive_expect_tx(bar(L::VFULL + s), L::kTileBytes);
                #pragma unroll
                for (int c = 0; c < L::kChunks; ++c)
                    tma_load_3d(sbase + L::kV + s * L::kTileBytes + c * L::kChunkBytes, &tm_v,
                                bar(L::VFULL + s), c * 64, j * kBN, bhk);
                v_uses[s] = use + 1;
            }
            // Drain: every load this thread issued has landed before the CTA may exit.
            mbar_drain(bar(L::QFULL), 0, kRoleProducer, 12);
            #pragma unroll
            for (int s = 0; s < NS; ++s) {
                if (k_uses[s] > 0) mbar_drain(bar(L::KFULL + s), (k_uses[s] - 1) & 1, kRoleProducer, 13);
                if (v_uses[s] > 0) mbar_drain(bar(L::VFULL + s), (v_uses[s] - 1) & 1, kRoleProducer, 14);
            }
        }
    } else if (warp == 5) {
        // =============================== MMA issuer ===============================
        if (lane == 0 && n_blocks > 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, true);
            const uint32_t q_addr = sbase + L::kQ;
            bool ok = mbar_wait(bar(L::QFULL), 0, limit, abort_flag, p.epoch, kRoleMma, 20);
            auto issue_pv = [&](int i) -> bool {
                const int vs = i % NS;
                if (!mbar_wait(bar(L::PFULL + (i & 1)), (i >> 1) & 1, limit, abort_flag, p.epoch, kRoleMma, 21)) return false;
                if (!mbar_wait(bar(L::VFULL + vs), (i / NS) & 1, limit, abort_flag, p.epoch, kRoleMma, 22)) return false;
                tc_fence_after();
                const uint32_t v_addr = sbase + L::kV + vs * L::kTileBytes;
                const uint32_t p_tmem = tmem + L::kColP + (i & 1) * 64;
                #pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    // V block rows kk*16 .. kk*16+15; 8-row groups 1024 B apart (SBO);
                    // the two 64-column halves of d are one chunk apart (LBO).
                    const uint64_t bdesc = smem_desc_sw128(v_addr + kk * 2048, L::kChunkBytes, 1024);
                    mma_ts(tmem + L::kColO, p_tmem + kk * 8, bdesc, kIdescO, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(L::VEMPTY + vs));
                mma_commit(bar(L::ODONE));
                return true;
            };
            for (int j = 0; ok && j < n_blocks; ++j) {
                const int ks = j % NS;
                if (!mbar_wait(bar(L::KFULL + ks), (j / NS) & 1, limit, abort_flag, p.epoch, kRoleMma, 23)) { ok = false; break; }
                tc_fence_after();
                const uint32_t k_addr = sbase + L::kK + ks * L::kTileBytes;
                const uint32_t s_tmem = tmem + L::kColS + (j & 1) * 128;
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // K-major 128-byte swizzle: 16 elements (32 B) per step inside a
                    // 64-element chunk; chunks are 16 KB apart.
                    const uint32_t off = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
                    const uint64_t adesc = smem_desc_sw128(q_addr + off, 16, 1024);
                    const uint64_t bdesc = smem_desc_sw128(k_addr + off, 16, 1024);
                    mma_ss(s_tmem, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(L::KEMPTY + ks));
                mma_commit(bar(L::SFULL + (j & 1)));
                if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
            }
            if (ok && issue_pv(n_blocks - 1)) mma_commit(bar(L::OFINAL));
            // Wait until every MMA this thread issued has completed before teardown.
            mma_commit(bar(L::MMAFIN));
            mbar_drain(bar(L::MMAFIN), 0, kRoleMma, 24);
        }
    } else {
        // ============================ softmax warps 0-3 ===========================
        const int row = warp * 32 + lane;
        const int q_idx = q0 + row;
        const uint32_t lane_tmem = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float c_log2 = p.scale_log2;
        float m_used = -INFINITY;  // running max (base-2, scaled), possibly stale by < tau
        float l_sum = 0.0f;        // running sum of exp2(t - m_used)
        bool ok = true;
        const float* mask_row = nullptr;
        if constexpr (HAS_MASK) {
            if (q_idx < p.Nq)
                mask_row = p.mask + static_cast<long long>(b) * p.msb + static_cast<long long>(h) * p.msh +
                           static_cast<long long>(q_idx) * p.msq;
        }

        for (int j = 0; j < n_blocks; ++j) {
            bool got = mbar_wait(bar(L::SFULL + (j & 1)), (j >> 1) & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 30);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[kBN];
            #pragma unroll
            for (int c = 0; c < kBN / 32; ++c)
                tmem_ld32(lane_tmem + L::kColS + (j & 1) * 128 + c * 32,
                          *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            tmem_wait_ld();
            float* s = reinterpret_cast<float*>(sr);
            const int j0 = j * kBN;

            float mx = -INFINITY;
            if constexpr (HAS_MASK) {
                // t = scale*log2e*qk + log2e*mask; masked keys -> -inf
                #pragma unroll
                // keys c >= lim are masked (past the end of K, or past the diagonal)
                int lim = mask_row != nullptr ? kv_len - j0 : 0;
                if (p.is_causal && q_idx - j0 + 1 < lim) lim = q_idx - j0 + 1;
                #pragma unroll
                for (int c = 0; c < kBN; ++c) {
                    const bool valid = c < lim;
                    const float mv = valid ? __ldg(mask_row + j0 + c) : 0.0f;
                    s[c] = valid ? fmaf(s[c], c_log2, mv * kLog2e) : -INFINITY;
                    mx = fmaxf(mx, s[c]);
                }
            } else {
                const bool boundary = (j0 + kBN > kv_len) || (p.is_causal && j0 + kBN - 1 > q0);
                if (boundary) {
                    int lim = kv_len - j0;
                    if (p.is_causal && q_idx - j0 + 1 < lim) lim = q_idx - j0 + 1;
                    #pragma unroll
                    for (int c = 0; c < kBN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
                }
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                #pragma unroll
                for (int c = 0; c < kBN; ++c) m4[c & 3] = fmaxf(m4[c & 3], s[c]);
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c_log2;
            }

            // Lazy correction: a row moves its reference max only when the block max
            // exceeds it by more than tau.  The TMEM load/store of O is warp-collective,
            // but each row applies its own decision (alpha = 1 exactly otherwise), so a
            // row's result never depends on the other rows of its warp.
            const bool need = mx > m_used + kLazyTau;
            if (__any_sync(0xffffffffu, need)) {
                const float m_new = need ? mx : m_used;
                const float alpha = !need ? 1.0f : (m_used == -INFINITY) ? 0.0f : ex2_approx(m_used - m_new);
                l_sum *= alpha;
                if (j > 0) {
                    // O holds sum_{i<j} P_i V_i once PV_{j-1} has completed.
                    got = mbar_wait(bar(L::ODONE), (j - 1) & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 31);
                    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                    tc_fence_after();
                    #pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(lane_tmem + L::kColO + c * 32, o);
                        tmem_wait_ld();
                        #pragma unroll
                        for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
                        tmem_st32(lane_tmem + L::kColO + c * 32, o);
                    }
                    tmem_wait_st();
                }
                m_used = m_new;
            }
            const float shift = (m_used == -INFINITY) ? 0.0f : m_used;

            float l4[4] = {0.f, 0.f, 0.f, 0.f};
            #pragma unroll
            for (int c = 0; c < kBN; ++c) {
                float e;
                if constexpr (HAS_MASK) e = ex2_approx(s[c] - shift);
                else e = ex2_approx(fmaf(s[c], c_log2, -shift));
                s[c] = e;
                l4[c & 3] += e;
            }
            l_sum += (l4[0] + l4[1]) + (l4[2] + l4[3]);

            uint32_t pk[kBN / 2];
            #pragma unroll
            for (int c = 0; c < kBN / 2; ++c) pk[c] = pack_bf16x2(s[2 * c], s[2 * c + 1]);
            const uint32_t p_tmem = lane_tmem + L::kColP + (j & 1) * 64;
            tmem_st32(p_tmem, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(p_tmem + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::PFULL + (j & 1)));
        }

        // ---------------------------------------------------------- epilogue
        if (ok && n_blocks > 0) {
            // A dedicated barrier: ODONE may still be a phase behind here (PV_{n-2}
            // need not have completed), and a parity test cannot tell.
            bool got = mbar_wait(bar(L::OFINAL), 0, limit, abort_flag, p.epoch, kRoleSoftmax, 32);
            ok = __all_sync(0xffffffffu, got);
            tc_fence_after();
        }
        const bool do_epilogue = __all_sync(0xffffffffu, ok && !*abort_flag);
        if (do_epilogue) {
            const float inv_l = l_sum > 0.0f ? 1.0f / l_sum : 0.0f;
            uint8_t* stage = smem + L::kQ;  // Q is dead once the last MMA has completed
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (n_blocks > 0) {
                    tmem_ld32(lane_tmem + L::kColO + c * 32, o);
                    tmem_wait_ld();
                } else {
                    #pragma unroll
                    for (int t = 0; t < 32; ++t) o[t] = 0u;
                }
                uint32_t w[16];
                #pragma unroll
                for (int t = 0; t < 16; ++t)
                    w[t] = pack_bf16x2(__uint_as_float(o[2 * t]) * inv_l, __uint_as_float(o[2 * t + 1]) * inv_l);
                const int chunk = (c * 32) / 64;
                const int unit0 = ((c * 32) % 64) / 8;
                #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int phys = (unit0 + u) ^ (row & 7);
                    uint4* dst = reinterpret_cast<uint4*>(stage + chunk * L::kChunkBytes + row * 128 + phys * 16);
                    *dst = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            }
            fence_proxy_async_smem();
            if (p.lse != nullptr && q_idx < p.Nq) {
                const float lse = l_sum > 0.0f ? (m_used + __log2f(l_sum)) * kLn2 : -INFINITY;
                p.lse[static_cast<long long>(bh) * p.Nq + q_idx] = lse;
            }
        }
        named_barrier_sync(1, 128);
        if (threadIdx.x == 0 && do_epilogue && !*abort_flag) {
            #pragma unroll
            for (int c = 0; c < L::kChunks; ++c)
                tma_store_3d(&tm_o, sbase + L::kQ + c * L::kChunkBytes, c * 64, q0, bh);
            bulk_commit_group();
            bulk_wait_group_read0();
        }
    }

    // ================================ teardown ================================
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
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
