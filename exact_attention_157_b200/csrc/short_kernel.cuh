// short_kernel.cuh -- exact attention forward pass for short key sequences
// (Nk <= 256, d = 64) on sm_100a: the short-sequence, memory-bound shapes (a
// ViT at 14 x 14 patches, text cross-attention with 77 keys).
//
// With at most 256 keys a whole score row fits in one tensor-memory
// accumulator, so the softmax needs no running rescale: S = Q K^T is computed
// in one product (N = the tile's key count rounded up to 16), the softmax reads
// the row once from tensor memory, 64 keys per step, and P V is one product.  This is the three steps of the definition per 128-row tile ("Flash
// Attention in a production Stable-Diffusion service", xxmr.cn/news/81028,
// section 2.3), tiled over queries as "FlashAttention technical analysis"
// (jsqmd.com/news/722897) section 2.2 tiles Q; the key block is the whole
// (short) key sequence.
//
// Work: one tile = 128 query rows of one (batch, query head).  Tiles are
// numbered head-major; persistent CTA c takes the contiguous range
// [c T / G, (c + 1) T / G), so consecutive tiles share their K/V head and K/V
// are loaded into shared memory once per run of tiles of one K/V head.
//
//   warps 0-3   softmax + epilogue of even tiles (tensor-memory slot 0)
//   warps 4-7   softmax + epilogue of odd tiles (slot 1)
//   warp 8      TMA producer: K and V of each run into one of two K/V buffers,
//               the Q tile into a ring of NQ stages
//   warp 9      TMEM owner and MMA issuer of slot 0: S(n), then P(n) V once P(n)
//               is stored, for the even tiles
//   warp 10     MMA issuer of slot 1 (odd tiles)
//   warp 11     idle (completes the third warpgroup)
//
// Tensor memory, slot s = columns [256 s, 256 s + 256): S in [0, N), P (bf16
// pairs) in [0, N / 2) written over the scores already read, O (64 fp32
// columns) in [128, 192) written by P V after the softmax has read every score.
// While one warpgroup runs its softmax, the other stores its output and the
// tensor cores compute the next S, so the two warpgroups run half a tile apart.
//
// Each slot's MMA warp issues S(n), PV(n), S(n + 2), PV(n + 2), ... for its
// tiles: S(n + 2) once the epilogue of tile n has read O out of the slot
// (OEMPTY).  With kShortEarlyS, an S whose columns stay below O (N <= 128) is
// issued right after PV(n) and only PV(n + 2) waits for that read; on B200 this
// measured slower (unet_cross 15.4 against 14.9 us), so it is off.  Commits release the Q stage (after S) and, with one arrival from
// each MMA warp, the K/V buffer (after the warp's last P V of the run; a warp
// with no tile in a run arrives once the run's K/V have landed, so that its
// arrival counts towards that use of the buffer).
//
// The two softmax warpgroups take turns (a token passed through an mbarrier):
// tile n + 1's exponentials start when tile n's are done, so the special-
// function units serve one tile at a time while the other warpgroup waits for
// its products or writes its output.
#pragma once

#include <type_traits>

#include "fwd_common.cuh"

namespace attn_sm100 {

constexpr int kShortThreads = 384;
constexpr bool kShortTurns = true;        // softmax warpgroups take turns (token)
constexpr bool kShortDirectStore = true;  // O rows stored from registers (else staged, TMA store)
constexpr bool kShortWarpStaged = true;   // direct stores: rows regrouped per warp through shared memory
constexpr bool kShortEarlyS = false;      // S(n + 2) before the epilogue of n when it fits below O (measured slower)
constexpr uint32_t kShortOCol = 128;      // first tensor-memory column of O within a slot
constexpr int kShortMaxKeys = 256;
constexpr int kShortMaxQ = 8;          // Q stages at most
constexpr int kShortTile = 128 * 128;  // one 128-row tile of 64 bf16 columns (16 KB)

struct ShortParams {
    int B, Hq, Hkv, Nq, Nk;
    int n_qt;         // 128-row tiles per (batch, head)
    int n_pad;        // Nk rounded up to 16: K/V rows loaded per head
    int nq_stages;    // Q ring stages (2..kShortMaxQ)
    int kv_bytes;     // bytes of one K (or V) buffer: n_pad * 128
    long long tiles;  // B * Hq * n_qt
    float scale_log2;
    int is_causal;
    const int32_t* key_lens;
    float* lse;
    void* out;
    unsigned long long timeout_ns;
    unsigned int epoch;
    FastDiv fd_qt, fd_hq, fd_group;
};

// Shared-memory layout (offsets from the 1024-aligned base).
struct SmemShort {
    int kv0, kv1, ost, q, bars, misc, bytes;
    __host__ __device__ static SmemShort make(int kv_bytes, int nq) {
        SmemShort s;
        s.kv0 = 0;                           // K then V of buffer 0
        s.kv1 = 2 * kv_bytes;                // K then V of buffer 1
        s.ost = 4 * kv_bytes;                // O staging, one 16 KB tile per warpgroup
        s.q = s.ost + 2 * kShortTile;        // Q ring
        s.bars = s.q + nq * kShortTile;
        s.misc = s.bars + 8 * kNumBars;
        s.bytes = s.misc + 16;
        return s;
    }
    // barrier indices
    static constexpr int QFULL = 0;                        // kShortMaxQ
    static constexpr int QEMPTY = kShortMaxQ;              // kShortMaxQ
    static constexpr int KVFULL = 2 * kShortMaxQ;          // 2
    static constexpr int KVEMPTY = KVFULL + 2;             // 2 (one arrival per MMA warp)
    static constexpr int SFULL = KVEMPTY + 2;              // 2 (per slot)
    static constexpr int PFULL = SFULL + 2;                // 2 (4 arrivals: one per warp)
    static constexpr int OFULL = PFULL + 2;                // 2
    static constexpr int OEMPTY = OFULL + 2;               // 2 (4 arrivals: one per warp)
    static constexpr int MMAFIN = OEMPTY + 2;              // 2 (per MMA warp)
    static constexpr int TURN = MMAFIN + 2;                // 2: warpgroup s may start its softmax (4 arrivals)
    static constexpr int kNumBars = TURN + 2;
};

// One tile's description, derived identically by every role.
struct ShortTile {
    int bh, bhk, q0, kv_len;
    int keys;   // keys the tile's rows may see: min(kv_len, causal ? q0 + 128 : Nk)
    int ncols;  // keys rounded up to 16: N of S = Q K^T, and the K extent of P V
    __device__ __forceinline__ bool empty() const { return keys <= 0; }
};

// The key length of batch entry b is read once per run of tiles of that entry
// (cb, ckv: the last entry read and its length), not once per tile.
__device__ __forceinline__ ShortTile short_tile(const ShortParams& p, long long t, int& cb, int& ckv, bool report) {
    ShortTile x;
    x.bh = fdiv(static_cast<int>(t), p.fd_qt);
    const int qi = static_cast<int>(t) - x.bh * p.n_qt;
    const int b = fdiv(x.bh, p.fd_hq);
    const int h = x.bh - b * p.Hq;
    x.bhk = b * p.Hkv + fdiv(h, p.fd_group);
    x.q0 = qi * 128;
    int kv = p.Nk;
    if (p.key_lens != nullptr) {
        if (b != cb) {
            cb = b;
            ckv = __ldg(p.key_lens + b);
            if (ckv < 0 || ckv > p.Nk) {
                if (report) record_error(kErrDevice, kRoleSoftmax, 40);
                ckv = ckv < 0 ? 0 : p.Nk;
            }
        }
        kv = ckv;
    }
    x.kv_len = kv;
    int keys = kv;
    if (p.is_causal && x.q0 + 128 < keys) keys = x.q0 + 128;
    x.keys = keys;
    x.ncols = (keys + 15) & ~15;
    return x;
}

// P V: O[128 x 64] (+)= P[128 x ncols] (tensor memory) V[ncols x 64] (shared),
// 16 keys per MMA, in batches of four, then the commits.
__device__ __forceinline__ void short_issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_addr, int ncols,
                                               uint32_t bar_a, uint32_t bar_b) {
    constexpr uint32_t kIdescO = idesc_bf16_f32(128, 64, true);
    constexpr int kVStep = 16 * 128 / 16;  // 16 keys of 128-byte rows, descriptor units
    const int steps = ncols >> 4;
    const uint64_t vd = smem_desc_sw128(v_addr, kShortTile, 1024);
    int k = 0;
    for (; k + 4 <= steps; k += 4) {
        const bool last = k + 4 == steps;
        mma_ts4_batch_warp<8, kVStep>(o_tmem, p_tmem + 8 * k, vd + static_cast<uint64_t>(k * kVStep), kIdescO,
                                      k > 0 ? 1u : 0u, last ? bar_a : 0u, last ? bar_b : 0u);
    }
    for (; k < steps; ++k) mma_ts_warp(o_tmem, p_tmem + 8 * k, vd + static_cast<uint64_t>(k * kVStep), kIdescO, k > 0);
    if (steps & 3) mma_commit2_warp(bar_a, bar_b);
}

__global__ void __launch_bounds__(kShortThreads, 1)
attn_fwd_short_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                      const ShortParams p) {
    using L = SmemShort;
    const SmemShort lay = SmemShort::make(p.kv_bytes, p.nq_stages);
    uint32_t dyn_smem;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
    if (dyn_smem < static_cast<uint32_t>(lay.bytes + 1024) || p.nq_stages < 2 || p.nq_stages > kShortMaxQ ||
        p.n_pad > kShortMaxKeys) {
        if (threadIdx.x == 0) record_error(kErrDevice, kRoleSoftmax, 41);
        return;
    }
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t sbase = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int NQ = p.nq_stages;
    auto bar = [&](int i) -> uint32_t { return sbase + lay.bars + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + lay.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + lay.misc + 4);

    const long long G = gridDim.x;
    // this CTA's tiles [t_begin, t_end)
    const long long t_begin = p.tiles * blockIdx.x / G;
    long long t_end = p.tiles * (blockIdx.x + 1) / G;
    int cb = -1, ckv = 0;  // key-length cache of this thread
    const uint64_t limit = p.timeout_ns;

    // Producer state.  The producer initialises the barriers and, before the
    // block-wide sync, already issues every load that needs no wait (the K/V of
    // the first two runs, the first NQ Q tiles), so that their latency overlaps
    // the tensor-memory allocation and the sync.
    long long pt = t_begin;     // next tile to load
    int pn = 0, pr = -1;        // Q tiles and K/V runs loaded
    int prev_bhk = -1;
    bool p_kv_done = false;     // the K/V of tile pt's run are issued
    bool p_ok = true;
    // Loads tiles from pt on; with may_wait false it stops at the first load that
    // would have to wait for a buffer.
    auto produce = [&](bool may_wait) {
        for (; p_ok && pt < t_end; ++pt, p_kv_done = false) {
            const ShortTile x = short_tile(p, pt, cb, ckv, false);
            if (x.empty()) continue;
            if (x.bhk != prev_bhk && !p_kv_done) {  // a new run: K and V of its head
                const int r = pr + 1;
                const int kb = r & 1;
                if (r >= 2) {
                    if (!may_wait) return;
                    if (!mbar_wait(bar(L::KVEMPTY + kb), ((r >> 1) - 1) & 1, limit, abort_flag, p.epoch,
                                   kRoleProducer, 42))
                        { p_ok = false; return; }
                }
                pr = r;
                const uint32_t kv = sbase + (kb ? lay.kv1 : lay.kv0);
                mbar_arrive_expect_tx(bar(L::KVFULL + kb), 2 * p.kv_bytes);
                tma_load_3d(kv, &tm_k, bar(L::KVFULL + kb), 0, 0, x.bhk);
                tma_load_3d(kv + p.kv_bytes, &tm_v, bar(L::KVFULL + kb), 0, 0, x.bhk);
                p_kv_done = true;
            }
            prev_bhk = x.bhk;
            const int st = pn % NQ;
            if (pn >= NQ) {
                if (!may_wait) return;
                if (!mbar_wait(bar(L::QEMPTY + st), ((pn / NQ) - 1) & 1, limit, abort_flag, p.epoch, kRoleProducer, 43))
                    { p_ok = false; return; }
            }
            mbar_arrive_expect_tx(bar(L::QFULL + st), kShortTile);
            tma_load_3d(sbase + lay.q + st * kShortTile, &tm_q, bar(L::QFULL + st), 0, x.q0, x.bh);
            ++pn;
        }
    };

    if (warp == 8 && lane == 0) {
        for (int q = 0; q < kShortMaxQ; ++q) {
            mbar_init(bar(L::QFULL + q), 1);
            mbar_init(bar(L::QEMPTY + q), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::KVFULL + s), 1);
            mbar_init(bar(L::KVEMPTY + s), 2);  // one arrival per MMA warp
            mbar_init(bar(L::SFULL + s), 1);
            mbar_init(bar(L::PFULL + s), 4);    // one arrival per softmax warp
            mbar_init(bar(L::OFULL + s), 1);
            mbar_init(bar(L::OEMPTY + s), 4);
            mbar_init(bar(L::MMAFIN + s), 1);
            mbar_init(bar(L::TURN + s), 4);
        }
        const bool aborted = launch_aborted(p.epoch);
        *abort_flag = aborted ? 1 : 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
        if (!aborted) produce(false);
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // none of the tiles if the launch was aborted before this CTA started
    if (__shfl_sync(0xffffffffu, *abort_flag, 0)) t_end = t_begin;

    if (warp == 8) {
        // ============================== TMA producer ==============================
        if (lane == 0) {
            produce(true);
            // every load issued has landed before the CTA may exit
            for (int st = 0; st < NQ && st < pn; ++st) {
                const int uses = (pn - 1 - st) / NQ + 1;  // loads into stage st
                mbar_drain(bar(L::QFULL + st), (uses - 1) & 1, kRoleProducer, 44);
            }
            for (int kb = 0; kb < 2 && kb <= pr; ++kb) {
                const int uses = (pr - kb) / 2 + 1;
                mbar_drain(bar(L::KVFULL + kb), (uses - 1) & 1, kRoleProducer, 45);
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ========================= MMA issuers (one per slot) =========================
        // Warp-uniform loop; one elected lane issues each batch and its commits.
        const int w = warp - 9;  // the slot, and the parity of the tiles served
        struct Ent {
            ShortTile x;
            int n, run;
            bool valid;
        };
        long long t_next = t_begin;
        int n_next = 0, run = -1, prev_bhk = -1;
        // the next tile with keys of this slot; tiles and K/V runs are counted over
        // the whole CTA, as the producer counts them
        auto next_own = [&]() -> Ent {
            Ent e;
            e.valid = false;
            while (t_next < t_end) {
                const ShortTile x = short_tile(p, t_next++, cb, ckv, false);
                if (x.empty()) continue;
                if (x.bhk != prev_bhk) { prev_bhk = x.bhk; ++run; }
                const int n = n_next++;
                if ((n & 1) != w) continue;
                e.x = x;
                e.n = n;
                e.run = run;
                e.valid = true;
                break;
            }
            return e;
        };
        int to_release = 0;  // K/V runs [0, to_release) released by this warp
        // runs below r in which this warp issued nothing: released once their K/V
        // have landed, so that the arrival counts towards that use of the buffer
        auto release_idle_runs = [&](int r) -> bool {
            for (; to_release < r; ++to_release) {
                if (!mbar_wait_warp(bar(L::KVFULL + (to_release & 1)), (to_release >> 1) & 1, limit, abort_flag,
                                    p.epoch, kRoleMma, 53))
                    return false;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::KVEMPTY + (to_release & 1)));
            }
            return true;
        };
        // S(n) = Q(n) K^T into the slot, then the SFULL commit and the Q stage released
        auto issue_s = [&](const Ent& e) -> bool {
            const int st = e.n % NQ;
            if (!mbar_wait_warp(bar(L::QFULL + st), (e.n / NQ) & 1, limit, abort_flag, p.epoch, kRoleMma, 46) ||
                !mbar_wait_warp(bar(L::KVFULL + (e.run & 1)), (e.run >> 1) & 1, limit, abort_flag, p.epoch, kRoleMma,
                                47))
                return false;
            tc_fence_after();
            const uint64_t qd = smem_desc_sw128(sbase + lay.q + st * kShortTile, 16, 1024);
            const uint64_t kd = smem_desc_sw128(sbase + ((e.run & 1) ? lay.kv1 : lay.kv0), 16, 1024);
            mma_ss_batch_warp<false, 4, 2, 2>(tmem + 256u * w, qd, kd, idesc_bf16_f32(128, e.x.ncols, false), 0u,
                                              bar(L::SFULL + w), bar(L::QEMPTY + st));
            return true;
        };
        bool ok = true;
        Ent cur = next_own();
        if (cur.valid) ok = release_idle_runs(cur.run) && issue_s(cur);
        bool o_held = false;  // O of this slot's previous tile not yet read out by its epilogue
        for (int i = 0; ok && cur.valid; ++i) {
            const Ent nxt = next_own();  // off the path from P to P V
            if (!mbar_wait_warp(bar(L::PFULL + w), i & 1, limit, abort_flag, p.epoch, kRoleMma, 48))
                { ok = false; break; }
            // P V overwrites O: the previous tile's epilogue must have read it
            if (o_held && !mbar_wait_warp(bar(L::OEMPTY + w), (i - 1) & 1, limit, abort_flag, p.epoch, kRoleMma, 49))
                { ok = false; break; }
            tc_fence_after();
            const bool last_of_run = !nxt.valid || nxt.run != cur.run;
            short_issue_pv(tmem + 256u * w + kShortOCol, tmem + 256u * w,
                           sbase + ((cur.run & 1) ? lay.kv1 : lay.kv0) + p.kv_bytes, cur.x.ncols, bar(L::OFULL + w),
                           last_of_run ? bar(L::KVEMPTY + (cur.run & 1)) : 0u);
            if (last_of_run) to_release = cur.run + 1;
            if (!nxt.valid) break;
            if (!release_idle_runs(nxt.run)) { ok = false; break; }
            // S(n + 2) goes into the slot at once when its columns stay clear of O
            // (products of one thread run in order, so P V has read P before S
            // overwrites it); a longer S waits until the epilogue has read O out
            o_held = kShortEarlyS && nxt.x.ncols <= static_cast<int>(kShortOCol);
            if (!o_held && !mbar_wait_warp(bar(L::OEMPTY + w), i & 1, limit, abort_flag, p.epoch, kRoleMma, 49))
                { ok = false; break; }
            if (!issue_s(nxt)) { ok = false; break; }
            cur = nxt;
        }
        // runs after this warp's last tile (the other slot's)
        if (ok) {
            while (next_own().valid) {}
            release_idle_runs(run + 1);
        }
        mma_commit_warp(bar(L::MMAFIN + w));
        mbar_drain(bar(L::MMAFIN + w), 0, kRoleMma, 50);
    } else if (warp < 8) {
        // =================== softmax + epilogue warpgroups (slots 0, 1) ===================
        const int s = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_tmem = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + 256u * s;
        const float c_log2 = p.scale_log2;
        const uint64_t c2 = pack_f32x2(c_log2, c_log2);
        uint8_t* stage = smem + lay.ost + s * kShortTile;
        bool ok = true;
        int n = 0;  // tiles with keys seen so far
        long long t_idx = 0;
        for (long long t = t_begin; t < t_end; ++t, ++t_idx) {
            const ShortTile x = short_tile(p, t, cb, ckv, threadIdx.x == 0);
            const int q = x.q0 + row;
            if (x.empty()) {
                // no key at all (key length 0): O = 0, LSE = -inf, written directly
                if ((t_idx & 1) == s && q < p.Nq && ok && !*abort_flag) {
                    const long long r = static_cast<long long>(x.bh) * p.Nq + q;
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + r * 64);
                    #pragma unroll
                    for (int v = 0; v < 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                    if (p.lse != nullptr) p.lse[r] = -INFINITY;
                }
                continue;
            }
            const int mine = n++;
            if ((mine & 1) != s) continue;
            const int u = mine >> 1;  // uses of this slot so far
            // Every warp of the warpgroup runs the named barriers of each of its tiles,
            // whether or not its waits succeeded, so that none is left waiting.
            bool tile_ok = ok;
            if (tile_ok) {
                const bool got = mbar_wait(bar(L::SFULL + s), u & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 51);
                tile_ok = __all_sync(0xffffffffu, got);
            }
            if (kShortTurns && tile_ok && (s == 1 || u > 0)) {
                // the other warpgroup's previous softmax is done
                const bool got = mbar_wait(bar(L::TURN + s), (s == 1 ? u : u - 1) & 1, limit, abort_flag, p.epoch,
                                           kRoleSoftmax, 54);
                tile_ok = __all_sync(0xffffffffu, got);
            }
            // keys of this row: j < lim are visible
            int lim = x.kv_len;
            if (p.is_causal && q + 1 < lim) lim = q + 1;
            const int ncols = x.ncols;
            const int n_chunks = (ncols + 31) >> 5;
            const bool dead = __all_sync(0xffffffffu, q >= p.Nq);  // the whole warp past the last row
            float m = -INFINITY, l_sum = 0.0f;
            if (tile_ok) {
                tc_fence_after();
                if (!dead) {
                    // One pass over the row, 64 keys per step.  The reference max m is the
                    // first step's maximum, raised only when a later step exceeds it by more than
                    // tau: then every stored P and the row sum are scaled by 2^-k, k an
                    // integer, which is exact (bf16 and fp32 keep their significands), so P
                    // carries one rounding like any other.  Exponents stay within 2^tau, far
                    // inside the range of bf16 P and the fp32 accumulators.
                    uint64_t acc0 = 0, acc1 = 0;
                    #pragma unroll 1
                    for (int g = 0; g < n_chunks; g += 2) {
                        // 64 keys per step: two 32-column loads, one wait
                        uint32_t sr[64];
                        const bool two = g + 1 < n_chunks;
                        tmem_ld32(lane_tmem + 32 * g, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                        if (two) tmem_ld32(lane_tmem + 32 * (g + 1), *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                        tmem_wait_ld();
                        float* sc = reinterpret_cast<float*>(sr);
                        const int j0 = 32 * g;
                        const int nk = two ? 64 : 32;  // columns loaded
                        if (j0 + nk > lim) {
                            #pragma unroll
                            for (int c = 0; c < 64; ++c) sc[c] = (j0 + c < lim) ? sc[c] : -INFINITY;
                        }
                        // four independent chains of 3-input maxima (a shorter dependency chain)
                        float x0 = fmax3(sc[0], sc[1], sc[2]), x1 = fmax3(sc[3], sc[4], sc[5]);
                        float x2 = fmax3(sc[6], sc[7], sc[8]), x3 = fmax3(sc[9], sc[10], sc[11]);
                        #pragma unroll
                        for (int c = 12; c < 28; c += 8) {
                            x0 = fmax3(x0, sc[c], sc[c + 1]);
                            x1 = fmax3(x1, sc[c + 2], sc[c + 3]);
                            x2 = fmax3(x2, sc[c + 4], sc[c + 5]);
                            x3 = fmax3(x3, sc[c + 6], sc[c + 7]);
                        }
                        x0 = fmax3(x0, sc[28], sc[29]);
                        x1 = fmax3(x1, sc[30], sc[31]);
                        if (two) {
                            #pragma unroll
                            for (int c = 32; c < 64; c += 8) {
                                x0 = fmax3(x0, sc[c], sc[c + 1]);
                                x1 = fmax3(x1, sc[c + 2], sc[c + 3]);
                                x2 = fmax3(x2, sc[c + 4], sc[c + 5]);
                                x3 = fmax3(x3, sc[c + 6], sc[c + 7]);
                            }
                        }
                        const float cmax = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3)) * c_log2;
                        if (g == 0) {
                            m = cmax == -INFINITY ? 0.0f : cmax;
                        } else if (__any_sync(0xffffffffu, cmax > m + kLazyTau)) {
                            const float kf = cmax > m + kLazyTau ? ceilf(cmax - m) : 0.0f;
                            const int k = static_cast<int>(kf);
                            const float a = k > 126 ? 0.0f : __int_as_float((127 - k) << 23);  // 2^-k exactly
                            m += kf;
                            acc0 = ffma2(acc0, pack_f32x2(a, a), 0ull);
                            acc1 = ffma2(acc1, pack_f32x2(a, a), 0ull);
                            for (int c0 = 0; c0 < 16 * g; c0 += 16) {
                                uint32_t pr[16];
                                tmem_ld16(lane_tmem + c0, pr);
                                tmem_wait_ld();
                                #pragma unroll
                                for (int v = 0; v < 16; ++v) {
                                    const float lo = __uint_as_float(pr[v] << 16) * a;
                                    const float hi = __uint_as_float(pr[v] & 0xffff0000u) * a;
                                    pr[v] = pack_bf16x2(lo, hi);
                                }
                                tmem_st16(lane_tmem + c0, pr);
                            }
                            tmem_wait_st();
                        }
                        const uint64_t ns2 = pack_f32x2(-m, -m);
                        uint32_t pk[32];
                        // exponentials of the first np pairs: the tile's key count rounded up
                        // to 16 bounds the pairs needed
                        auto exps = [&](auto np_c) {
                            constexpr int np = decltype(np_c)::value;
                            #pragma unroll
                            for (int c = 0; c < np; ++c) {
                                const uint64_t xv = ffma2(pack_f32x2(sc[2 * c], sc[2 * c + 1]), c2, ns2);
                                const float e0 = ex2_approx(lo_f32(xv)), e1 = ex2_approx(hi_f32(xv));
                                if (c & 1) acc1 = fadd2(acc1, pack_f32x2(e0, e1));
                                else acc0 = fadd2(acc0, pack_f32x2(e0, e1));
                                pk[c] = pack_bf16x2(e0, e1);
                            }
                            #pragma unroll
                            for (int c = np; c < 32; ++c) pk[c] = 0u;
                        };
                        const int left = ncols - j0;  // columns of this step the products read
                        if (left >= 64) exps(std::integral_constant<int, 32>{});
                        else if (left >= 48) exps(std::integral_constant<int, 24>{});
                        else if (left >= 32) exps(std::integral_constant<int, 16>{});
                        else exps(std::integral_constant<int, 8>{});
                        tmem_st32(lane_tmem + 16 * g, pk);
                    }
                    const uint64_t acc = fadd2(acc0, acc1);
                    l_sum = lo_f32(acc) + hi_f32(acc);
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar(L::PFULL + s));
                    if (kShortTurns) mbar_arrive(bar(L::TURN + (s ^ 1)));  // the other warpgroup's turn
                }
                // epilogue: O / l once P V is complete
                const bool got_o = mbar_wait(bar(L::OFULL + s), u & 1, limit, abort_flag, p.epoch, kRoleSoftmax, 52);
                tile_ok = __all_sync(0xffffffffu, got_o);
            }
            ok = tile_ok;
            const float inv_l = l_sum > 0.0f ? 1.0f / l_sum : 0.0f;
            if constexpr (kShortDirectStore) {
                if (tile_ok) {
                    tc_fence_after();
                    uint32_t o[64];
                    tmem_ld32(lane_tmem + kShortOCol, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                    tmem_ld32(lane_tmem + kShortOCol + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(L::OEMPTY + s));  // O may be overwritten now
                    const long long r = static_cast<long long>(x.bh) * p.Nq + q;
                    if constexpr (kShortWarpStaged) {
                        // the warp's 32 rows (4 KB) pass through shared memory (16-byte
                        // units swizzled by row, no bank conflicts), then each store
                        // instruction writes four whole consecutive rows (512 bytes)
                        uint8_t* ws = stage + (warp & 3) * 4096;
                        #pragma unroll
                        for (int v = 0; v < 8; ++v)
                            *reinterpret_cast<uint4*>(ws + lane * 128 + ((v ^ (lane & 7)) << 4)) = make_uint4(
                                pack_bf16x2(__uint_as_float(o[8 * v]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l));
                        __syncwarp();
                        const int q_warp = x.q0 + (warp & 3) * 32;  // the warp's first row
                        const int cu = lane & 7;                     // 16-byte unit of the row
                        if (!*abort_flag) {
                            #pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int rr = 4 * j + (lane >> 3);  // row within the warp
                                const uint4 val = *reinterpret_cast<const uint4*>(ws + rr * 128 + ((cu ^ (rr & 7)) << 4));
                                if (q_warp + rr < p.Nq) {
                                    const long long g = static_cast<long long>(x.bh) * p.Nq + q_warp + rr;
                                    reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + g * 64)[cu] = val;
                                }
                            }
                        }
                        __syncwarp();  // the buffer is written again only after every lane has read it
                        if (q < p.Nq && !*abort_flag && p.lse != nullptr)
                            p.lse[r] = l_sum > 0.0f ? (m + __log2f(l_sum)) * kLn2 : -INFINITY;
                    } else if (q < p.Nq && !*abort_flag) {
                        // each thread writes its own 128-byte row of O from registers
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + r * 64);
                        #pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_uint4(
                                pack_bf16x2(__uint_as_float(o[8 * v]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l));
                        if (p.lse != nullptr) p.lse[r] = l_sum > 0.0f ? (m + __log2f(l_sum)) * kLn2 : -INFINITY;
                    }
                }
            } else {
                uint32_t o[64];
                if (tile_ok) {
                    tc_fence_after();
                    tmem_ld32(lane_tmem + kShortOCol, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                    tmem_ld32(lane_tmem + kShortOCol + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(L::OEMPTY + s));  // O may be overwritten now
                }
                // the previous tile's TMA store must have read the staging buffer
                if ((threadIdx.x & 127) == 0) bulk_wait_group_read0();
                named_barrier_sync(1 + s, 128);
                if (tile_ok) {
                    #pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const int phys = v ^ (row & 7);  // 128-byte swizzle of the 16-byte units
                        uint4* dst = reinterpret_cast<uint4*>(stage + row * 128 + phys * 16);
                        *dst = make_uint4(
                            pack_bf16x2(__uint_as_float(o[8 * v]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l),
                            pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l),
                            pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l),
                            pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l));
                    }
                    fence_proxy_async_smem();
                    if (p.lse != nullptr && q < p.Nq)
                        p.lse[static_cast<long long>(x.bh) * p.Nq + q] =
                            l_sum > 0.0f ? (m + __log2f(l_sum)) * kLn2 : -INFINITY;
                }
                named_barrier_sync(1 + s, 128);
                // (a failed wait anywhere in the CTA sets the abort flag: no store then)
                if ((threadIdx.x & 127) == 0 && !*abort_flag) {
                    tma_store_3d(&tm_o, smem_u32(stage), 0, x.q0, x.bh);
                    bulk_commit_group();
                }
            }
        }
    }

    // ================================ teardown ================================
    if (warp < 8 && (threadIdx.x & 127) == 0) bulk_wait_group_read0();
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn_sm100
