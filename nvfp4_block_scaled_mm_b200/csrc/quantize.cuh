// NVFP4 quantizer: bf16 [rows, K] -> E2M1 codes (two per byte, element 2j in the low nibble of
// byte j) and UE4M3 block scales over 16 K-elements in the 128x4 swizzled layout, rows padded to
// 128 (sm_100a).
//
// The mm_nvfp4_lora page names fp4_quantize as the producer of its a / a_sf operands and folds a
// per-tensor global scale gs into alpha (Parameters: alpha = alpha_base / (a_global_scale *
// b_global_scale)), but gives no rule.  This kernel computes, per 16-element block, in float32:
//     amax = max |x|;  sf = E4M3_rne_satfinite((amax * gs) / 6);  inv = gs / value(sf);
//     code = E2M1_rne_satfinite(x * inv)   (a zero scale gives +0 codes),
// and writes 0 into the scale bytes of the padded rows.  The conversions are the hardware's
// (cvt.rn.satfinite.e4m3x2 / .e2m1x2: round to nearest even, saturate to the largest finite).
//
// HBM-bound: 2 bytes read and 0.5 + 1/16 written per element.  One thread per 16-element block
// (two 16-byte loads, one 8-byte store of codes); a warp covers 32 consecutive blocks of a row,
// so its loads and code stores are contiguous, and four lanes combine their scale bytes into one
// 4-byte store (the 4 K-groups of a scale atom row are adjacent in the swizzled layout).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace nvfp4lora {

constexpr int kQuantThreads = 256;

// float32 >= 0 -> E4M3 byte (round to nearest even, saturating at 448)
__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float v) {
    uint16_t two;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(0.0f), "f"(v));
    return two & 0xFFu;
}

// E4M3 byte -> its value as float32 (exact)
__device__ __forceinline__ float e4m3_value(uint32_t byte) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)byte));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// two float32 -> one byte of E2M1 codes: lo in bits 3..0, hi in bits 7..4
__device__ __forceinline__ uint32_t e2m1x2_rn_satfinite(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(out) : "f"(hi), "f"(lo));
    return out;
}

// One 16-element block: amax, scale byte, 16 codes (8 bytes); `w` holds the block's 16 bf16.
__device__ __forceinline__ uint32_t quantize_block(const uint4 w0, const uint4 w1, float gs, uint2& packed_out) {
    const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float v[16];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(wv[i] << 16);
        v[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
    }
    const uint32_t sfb = e4m3_rn_satfinite(__fdiv_rn(__fmul_rn(amax, gs), 6.0f));
    uint32_t packed[2] = {0u, 0u};
    const float sfv = e4m3_value(sfb);
    if (sfv > 0.0f) {
        const float inv = __fdiv_rn(gs, sfv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t byte = e2m1x2_rn_satfinite(__fmul_rn(v[2 * i], inv), __fmul_rn(v[2 * i + 1], inv));
            packed[i >> 2] |= byte << ((i & 3) * 8);
        }
    }
    packed_out = make_uint2(packed[0], packed[1]);
    return sfb;
}

// One thread per 16-element block per step; launch bounds for 8 resident CTAs (64 warps) per SM,
// so that enough loads are in flight to cover the memory latency.
__global__ void __launch_bounds__(kQuantThreads, 8)
quantize_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, const float* __restrict__ gs_ptr,
                uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
    const float gs = *gs_ptr;
    const int64_t nb = k / 16;                               // blocks per row (a multiple of 4)
    const int64_t rows_p = (rows + 127) / 128 * 128;
    const int64_t total = rows_p * nb;                       // a multiple of 4
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;  // a multiple of 32
    const int lane = threadIdx.x & 31;
    // every lane runs the same number of iterations, so the shuffles below see a full warp
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total; base += stride) {
        const int64_t blk = base + lane;
        const bool live = blk < total;
        const int64_t r = live ? blk / nb : 0;
        const int64_t c = live ? blk % nb : 0;
        uint32_t sfb = 0;
        if (live && r < rows) {
            const uint4* src = reinterpret_cast<const uint4*>(x + r * k + c * 16);
            uint2 packed;
            sfb = quantize_block(__ldg(src), __ldg(src + 1), gs, packed);
            *reinterpret_cast<uint2*>(codes + r * (k / 2) + c * 8) = packed;
        }
        // four consecutive blocks of a row: one 4-byte store into the swizzled scale atom
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, sfb, 1);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, sfb, 2);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, sfb, 3);
        if (live && (lane & 3) == 0) {
            const int64_t off = ((r / 128) * (nb / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4;
            *reinterpret_cast<uint32_t*>(sf + off) = sfb | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
    }
}

}  // namespace nvfp4lora
