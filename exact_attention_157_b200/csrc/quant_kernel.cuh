// quant_kernel.cuh -- FP8 E4M3 block quantisation of bf16 rows on the device:
// one fp32 scale per 128-row block of every head, scale = block amax / 448,
// code = round-to-nearest-even E4M3 of x / scale (the division correctly
// rounded in fp32).  "FlashAttention technical analysis"
// (jsqmd.com/news/722897), sections 4.2 (FP8 inputs with block quantisation)
// and 6.3 (each block keeps its own scale factor).
#pragma once

#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int kQuantRows = 128;    // rows per block, the FP8 attention path's tile height
constexpr int kQuantThreads = 256; // two threads per row, each half of the row

// One CTA per (head, 128-row block).  Reads the block once into registers,
// reduces |x| to the block maximum, writes the scale and the codes.  HBM-bound:
// 2 bytes in and 1 byte out per element.
template <int D>
__global__ void __launch_bounds__(kQuantThreads)
attn_quantize_e4m3_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ codes, float* __restrict__ scales,
                          int N, int nb) {
    constexpr int kHalf = D / 2;          // elements per thread
    constexpr int kVec = kHalf * 2 / 16;  // 16-byte loads per thread
    __shared__ float warp_max[kQuantThreads / 32];
    const int head_blk = blockIdx.x;
    const long long head = head_blk / nb;
    const int blk = head_blk - static_cast<int>(head) * nb;
    const int r = blk * kQuantRows + (threadIdx.x >> 1);
    const int half = threadIdx.x & 1;
    const bool valid = r < N;
    const long long off = (head * N + r) * D + half * kHalf;
    uint4 v[kVec];
    float amax = 0.0f;
    if (valid) {
        const uint4* src = reinterpret_cast<const uint4*>(x + off);
        #pragma unroll
        for (int i = 0; i < kVec; ++i) v[i] = __ldg(src + i);
        #pragma unroll
        for (int i = 0; i < kVec; ++i) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            #pragma unroll
            for (int j = 0; j < 4; ++j) {
                amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
                amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xffff0000u)));
            }
        }
    }
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    float m = warp_max[0];
    #pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, warp_max[i]);
    const float scale = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
    if (threadIdx.x == 0) scales[head * nb + blk] = scale;
    if (!valid) return;
    uint32_t out[kHalf / 4];
    #pragma unroll
    for (int i = 0; i < kVec; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        float f[8];
        #pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = __uint_as_float(w[j] << 16);
            f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
        }
        #pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = fminf(fmaxf(__fdiv_rn(f[j], scale), -448.0f), 448.0f);
        out[2 * i] = pack_e4m3x4(f[0], f[1], f[2], f[3]);
        out[2 * i + 1] = pack_e4m3x4(f[4], f[5], f[6], f[7]);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + off);
    #pragma unroll
    for (int i = 0; i < kHalf / 16; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
}

}  // namespace attn_sm100
