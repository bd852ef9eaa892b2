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
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Roles for error reporting.
enum : unsigned int { kRoleSoftmax = 1, kRoleProducer = 2, kRoleMma = 3, kRoleSelftest = 9 };

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
    unsigned long long timeout_ns;
    unsigned int epoch;  // launch id for the launch-wide abort (never 0)
};

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
