// fwd_kernel_pp.cuh -- exact attention forward pass for sm_100a, two query tiles
// per CTA ("ping-pong").
//
// A CTA owns 256 query rows of one (batch, query head): tile A = rows q0..q0+127,
// tile B = rows q0+128..q0+255.  Both tiles share every K/V block, so K/V are
// read from shared memory once per 256 rows.
//
//   warps 0-3   softmax of tile A (thread = row = TMEM lane)
//   warps 4-7   softmax of tile B
//   warp 8      TMA producer: Q_A, Q_B once, then K_0, V_0, K_1, V_1, ... into
//               one ring of NSLOT shared-memory slots (128-byte swizzle, no
//               multicast), in the order the MMAs consume them
//   warps 10-11 idle (they complete the third warpgroup that setmaxnreg needs)
//   warp 9      TMEM owner and MMA issuer (one thread), order
//                 S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) S_A(2) ...
//               so that while the softmax of one tile runs, the tensor cores
//               work on the other tile (two MMAs of cover each way)
//
// TMEM: S_A cols [0,128), S_B [128,256), O_A [256,256+D), O_B [256+D,256+2D).
// P_t (bf16 pairs, 64 cols) overwrites the first half of S_t once the softmax
// has read S_t; S_t(j+1) is issued after PV_t(j) by the same thread, and
// tcgen05.mma operations of one thread execute in issue order.  Because S_t(j)
// is issued after PV_t(j-1), S_t(j) complete implies O_t = sum_{i<j} P_i V_i,
// so the softmax may rescale O_t right away, without another barrier.
//
// Online softmax in base 2 with the scale folded into the FMA and lazy
// rescaling ("FlashAttention technical analysis", jsqmd.com/news/722897,
// sections 2.2 and 4.1); one final normalisation; LSE = (m + log2 l) ln 2.
#pragma once

#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int kPPThreads = 384;  // 12 warps = 3 warpgroups
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512);
// the TMA/MMA warpgroup gives back to 72 and the two softmax warpgroups take
// 216: 2 x 128 x 216 + 128 x 72 = 64512, exactly the launch total.
constexpr int kRegsSoftmax = 216;
constexpr int kRegsControl = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kPPThreads * 168, "register split");

template <int D, int NSLOT>
struct SmemPP {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = 128 * 128;
    static constexpr int kTileBytes = kChunks * kChunkBytes;  // 128 rows x D bf16
    static constexpr int kQ = 0;                              // Q_A, then Q_B
    static constexpr int kRing = 2 * kTileBytes;
    static constexpr int kBars = kRing + NSLOT * kTileBytes;
    // barrier indices
    static constexpr int QFULL = 0;
    static constexpr int FULL = 1;                 // NSLOT
    static constexpr int EMPTY = 1 + NSLOT;        // NSLOT
    static constexpr int SFULL = 1 + 2 * NSLOT;    // 2 (per tile)
    static constexpr int PFULL = 3 + 2 * NSLOT;    // 2
    static constexpr int OFINAL = 5 + 2 * NSLOT;   // 2
    static constexpr int MMAFIN = 7 + 2 * NSLOT;
    static constexpr int kNumBars = 8 + 2 * NSLOT;
    static constexpr int kMisc = kBars + 8 * kNumBars;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kColO = 256;
    static_assert(kColO + 2 * D <= kTmemCols, "TMEM budget");
    static_assert(kAlloc <= 232448, "shared memory budget");
};

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

template <int D, int NSLOT, bool HAS_MASK>
__global__ void __launch_bounds__(kPPThreads, 1)
attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdParams p) {
    using L = SmemPP<D, NSLOT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t sbase = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- CTA coordinates: p.n_qtiles counts 256-row CTA tiles here
    const int bh = blockIdx.x / p.n_qtiles;
    int qt = blockIdx.x % p.n_qtiles;
    if (p.is_causal) qt = p.n_qtiles - 1 - qt;  // heavier causal tiles of a head first
    const int b = bh / p.Hq;
    const int h = bh - b * p.Hq;
    const int bhk = b * p.Hkv + h / p.group;
    const int q0 = qt * 2 * kBM;
    const bool tile_b_valid = q0 + kBM < p.Nq;
    int kv_len = p.Nk;
    if (p.key_lens != nullptr) {
        kv_len = p.key_lens[b];
        if (kv_len < 0 || kv_len > p.Nk) {
            if (threadIdx.x == 0) record_error(kErrDevice, kRoleSoftmax, 1);
            kv_len = kv_len < 0 ? 0 : p.Nk;
        }
    }
    // key blocks per tile: causal tiles stop at their diagonal block
    int n_t[2];
    #pragma unroll
    for (int t = 0; t < 2; ++t) {
        int end = kv_len;
        if (p.is_causal && q0 + (t + 1) * kBM < end) end = q0 + (t + 1) * kBM;
        n_t[t] = (end + kBN - 1) / kBN;
    }
    if (!tile_b_valid) n_t[1] = 0;

    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(L::QFULL), 1);
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(bar(L::FULL + s), 1);
            mbar_init(bar(L::EMPTY + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(L::SFULL + t), 1);
            mbar_init(bar(L::PFULL + t), 128);
            mbar_init(bar(L::OFINAL + t), 1);
        }
        mbar_init(bar(L::MMAFIN), 1);
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
    if (*abort_flag) { n_t[0] = 0; n_t[1] = 0; }
    n_t[0] = __shfl_sync(0xffffffffu, n_t[0], 0);
    n_t[1] = __shfl_sync(0xffffffffu, n_t[1], 0);
    const int n_max = n_t[0] > n_t[1] ? n_t[0] : n_t[1];

    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(kRegsControl));
      if (warp >= 10) {
        // idle warps
      } else if (warp == 8) {
        // ============================== TMA producer ==============================
        if (lane == 0 && n_max > 0) {
            int uses[NSLOT];
            #pragma unroll
            for (int s = 0; s < NSLOT; ++s) uses[s] = 0;
            const int n_q_tiles = tile_b_valid ? 2 : 1;
            mbar_arrive_expect_tx(bar(L::QFULL), n_q_tiles * L::kTileBytes);
            for (int t = 0; t < n_q_tiles; ++t) {
                #pragma unroll
                for (int c = 0; c < L::kChunks; ++c)
                    tma_load_3d(sbase + L::kQ + t * L::kTileBytes + c * L::kChunkBytes, &tm_q, bar(L::QFULL),
                                c * 64, q0 + t * kBM, bh);
            }
            const int n_loads = 2 * n_max;  // K_0, V_0, K_1, V_1, ...
            for (int i = 0; i < n_loads; ++i) {
                const int s = i % NSLOT;
                const int use = i / NSLOT;
                if (use > 0 &&
                    !mbar_wait(bar(L::EMPTY + s), (use - 1) & 1, limit, abort_flag, p.epoch, kRoleProducer, 10))
                    break;
                const CUtensorMap* map = (i & 1) ? &tm_v : &tm_k;
                mbar_arrive_expect_tx(bar(L::FULL + s), L::kTileBytes);
                #pragma unroll
                for (int c = 0; c < L::kChunks; ++c)
                    tma_load_3d(sbase + L::kRing + s * L::kTileBytes + c * L::kChunkBytes, map, bar(L::FULL + s),
                                c * 64, (i >> 1) * kBN, bhk);
                uses[s] = use + 1;
            }
            mbar_drain(bar(L::QFULL), 0, kRoleProducer, 12);
            #pragma unroll
            for (int s = 0; s < NSLOT; ++s)
                if (uses[s] > 0) mbar_drain(bar(L::FULL + s), (uses[s] - 1) & 1, kRoleProducer, 13);
        }
    } else if (warp == 9) {
        // =============================== MMA issuer ===============================
        if (lane == 0 && n_max > 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, true);
            auto slot_of = [](int i) { return i % NSLOT; };
            auto wait_full = [&](int i, unsigned site) -> bool {
                return mbar_wait(bar(L::FULL + slot_of(i)), (i / NSLOT) & 1, limit, abort_flag, p.epoch, kRoleMma, site);
            };
            auto issue_s = [&](int t, int j) {
                const uint32_t q_addr = sbase + L::kQ + t * L::kTileBytes;
                const uint32_t k_addr = sbase + L::kRing + slot_of(2 * j) * L::kTileBytes;
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
                    mma_ss(tmem + t * 128, smem_desc_sw128(q_addr + off, 16, 1024),
                           smem_desc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(L::SFULL + t));
            };
            auto issue_pv = [&](int t, int j) {
                const uint32_t v_addr = sbase + L::kRing + slot_of(2 * j + 1) * L::kTileBytes;
                const uint32_t o_tmem = tmem + L::kColO + t * D;
                const uint32_t p_tmem = tmem + t * 128;
                #pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(o_tmem, p_tmem + kk * 8, smem_desc_sw128(v_addr + kk * 2048, L::kChunkBytes, 1024),
                           kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
            };
            bool ok = mbar_wait(bar(L::QFULL), 0, limit, abort_flag, p.epoch, kRoleMma, 20) && wait_full(0, 21);
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (n_t[t] > 0) issue_s(t, 0);
                mma_commit(bar(L::EMPTY + slot_of(0)));  // K_0 released once both S(0) complete
            }
            for (int j = 0; ok && j < n_max; ++j) {
                bool v_ready = false, k_next_ready = false;
                for (int t = 0; t < 2 && ok; ++t) {
                    if (j >= n_t[t]) continue;
                    if (!mbar_wait(bar(L::PFULL + t), j & 1, limit, abort_flag, p.epoch, kRoleMma, 22)) { ok = false; break; }
                    if (!v_ready) {
                        if (!wait_full(2 * j + 1, 23)) { ok = false; break; }
                        v_ready = true;
                    }
                    tc_fence_after();
                    issue_pv(t, j);
                    if (j + 1 < n_t[t]) {
                        if (!k_next_ready) {
                            if (!wait_full(2 * j + 2, 24)) { ok = false; break; }
                            k_next_ready = true;
                            tc_fence_after();
                        }
                        issue_s(t, j + 1);
                    } else {
                        mma_commit(bar(L::OFINAL + t));
                    }
                }
                if (!ok) break;
                mma_commit(bar(L::EMPTY + slot_of(2 * j + 1)));      // V_j: both PV(j) issued above
                // K_{j+1}: the tile with n_t = n_max uses every block, so k_next_ready
                // holds exactly when j + 1 < n_max (each load is released once).
                if (k_next_ready) mma_commit(bar(L::EMPTY + slot_of(2 * j + 2)));
            }
            mma_commit(bar(L::MMAFIN));
            mbar_drain(bar(L::MMAFIN), 0, kRoleMma, 25);
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(kRegsSoftmax));
        // ======================= softmax warpgroups (tiles A, B) ===================
        const int t = warp >> 2;             // tile
        const int row = (warp & 3) * 32 + lane;
        const int q_idx = q0 + t * kBM + row;
        const int q0_t = q0 + t * kBM;
        const int n_blocks = n_t[t];
        const uint32_t lane_tmem = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t s_tmem = lane_tmem + t * 128;
        const uint32_t o_tmem = lane_tmem + L::kColO + t * D;
        const float c_log2 = p.scale_log2;
        const uint64_t c2 = pack_f32x2(c_log2, c_log2);
        float m_used = -INFINITY;
        float l_sum = 0.0f;
        bool ok = true;
        const float* mask_row = nullptr;
        if constexpr (HAS_MASK) {
            if (q_idx < p.Nq)
                mask_row = p.mask + static_cast<long long>(b) * p.msb + static_cast<long long>(h) * p.msh +
                           static_cast<long long>(q_idx) * p.msq;
        }

        for (int j = 0; j < n_blocks; ++j) {
            bool got = mbar_wait(bar(L::SFULL + t), j & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 30);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[kBN];
            #pragma unroll
            for (int c = 0; c < kBN / 32; ++c)
                tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            tmem_wait_ld();
            float* s = reinterpret_cast<float*>(sr);
            const int j0 = j * kBN;

            float mx;
            if constexpr (HAS_MASK) {
                mx = -INFINITY;
                #pragma unroll
                for (int c = 0; c < kBN; ++c) {
                    const int key = j0 + c;
                    const bool valid = mask_row != nullptr && key < kv_len && !(p.is_causal && key > q_idx);
                    const float mv = valid ? __ldg(mask_row + key) : 0.0f;
                    s[c] = valid ? fmaf(s[c], c_log2, mv * kLog2e) : -INFINITY;
                    mx = fmaxf(mx, s[c]);
                }
            } else {
                if ((j0 + kBN > kv_len) || (p.is_causal && j0 + kBN - 1 > q0_t)) {
                    #pragma unroll
                    for (int c = 0; c < kBN; ++c) {
                        const int key = j0 + c;
                        if (key >= kv_len || (p.is_causal && key > q_idx)) s[c] = -INFINITY;
                    }
                }
                float ma = fmax3(s[0], s[1], s[2]);
                float mb = fmax3(s[3], s[4], s[5]);
                #pragma unroll
                for (int c = 6; c + 3 < kBN; c += 4) {
                    ma = fmax3(ma, s[c], s[c + 1]);
                    mb = fmax3(mb, s[c + 2], s[c + 3]);
                }
                mx = fmax3(ma, mb, s[kBN - 2]);
                mx = fmaxf(mx, s[kBN - 1]) * c_log2;
            }

            // Lazy correction, decided per row (see the single-tile kernel).  O_t holds
            // sum_{i<j} P_i V_i here: S_t(j) was issued after PV_t(j-1).  The TMEM
            // rescale of O_t itself is done after P_t is stored (fewer live registers);
            // it only has to precede the PFULL arrive that lets PV_t(j) start.
            const bool need = mx > m_used + kLazyTau;
            const bool warp_rescale = __any_sync(0xffffffffu, need) && j > 0;
            float alpha = 1.0f;
            if (need) {
                alpha = (m_used == -INFINITY) ? 0.0f : ex2_approx(m_used - mx);
                l_sum *= alpha;
                m_used = mx;
            }
            const float shift = (m_used == -INFINITY) ? 0.0f : m_used;
            const uint64_t nshift2 = pack_f32x2(-shift, -shift);

            uint64_t acc0 = 0, acc1 = 0;  // two packed partial sums
            uint32_t pk[kBN / 2];
            #pragma unroll
            for (int c = 0; c < kBN / 2; ++c) {
                float e0, e1;
                if constexpr (HAS_MASK) {
                    e0 = ex2_approx(s[2 * c] - shift);
                    e1 = ex2_approx(s[2 * c + 1] - shift);
                } else {
                    const uint64_t x = ffma2(pack_f32x2(s[2 * c], s[2 * c + 1]), c2, nshift2);
                    e0 = ex2_approx(lo_f32(x));
                    e1 = ex2_approx(hi_f32(x));
                }
                if (c & 1) acc1 = fadd2(acc1, pack_f32x2(e0, e1));
                else acc0 = fadd2(acc0, pack_f32x2(e0, e1));
                pk[c] = pack_bf16x2(e0, e1);
            }
            const uint64_t acc = fadd2(acc0, acc1);
            l_sum += lo_f32(acc) + hi_f32(acc);

            tmem_st32(s_tmem, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(s_tmem + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            if (warp_rescale) {
                #pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(o_tmem + c * 32, o);
                    tmem_wait_ld();
                    #pragma unroll
                    for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
                    tmem_st32(o_tmem + c * 32, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::PFULL + t));
        }

        // ---------------------------------------------------------- epilogue
        if (ok && n_blocks > 0) {
            bool got = mbar_wait(bar(L::OFINAL + t), 0, limit, abort_flag, p.epoch, kRoleSoftmax, 32);
            ok = __all_sync(0xffffffffu, got);
            tc_fence_after();
        }
        const bool do_epilogue = __all_sync(0xffffffffu, ok && !*abort_flag) && q0_t < p.Nq;
        if (do_epilogue) {
            const float inv_l = l_sum > 0.0f ? 1.0f / l_sum : 0.0f;
            uint8_t* stage = smem + L::kQ + t * L::kTileBytes;  // Q_t is dead after OFINAL_t
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (n_blocks > 0) {
                    tmem_ld32(o_tmem + c * 32, o);
                    tmem_wait_ld();
                } else {
                    #pragma unroll
                    for (int u = 0; u < 32; ++u) o[u] = 0u;
                }
                uint32_t w[16];
                #pragma unroll
                for (int u = 0; u < 16; ++u)
                    w[u] = pack_bf16x2(__uint_as_float(o[2 * u]) * inv_l, __uint_as_float(o[2 * u + 1]) * inv_l);
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
        named_barrier_sync(1 + t, 128);
        if ((threadIdx.x & 127) == 0 && do_epilogue && !*abort_flag) {
            #pragma unroll
            for (int c = 0; c < L::kChunks; ++c)
                tma_store_3d(&tm_o, sbase + L::kQ + t * L::kTileBytes + c * L::kChunkBytes, c * 64, q0_t, bh);
            bulk_commit_group();
            bulk_wait_group_read0();
        }
    }

    // ================================ teardown ================================
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn_sm100
