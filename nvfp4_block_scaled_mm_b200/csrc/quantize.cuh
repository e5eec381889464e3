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
// 4-byte store (the 4 K-groups of a scale atom row are adjacent in the swizzled layout).  The
// instruction count per block is kept low so that issue does not limit the kernel before HBM does:
// the amax is a packed bf16x2 max over the absolute values, gs / value(sf) comes from a per-CTA
// table of the 126 positive E4M3 values (the same division, done once per value), (amax*gs)/6 is
// the FMA-corrected quotient below, the 16 scalings are packed f32x2 multiplies, and each thread
// steps its (row, block) position by the grid stride instead of dividing every iteration.
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

// eight float32 -> four bytes of E2M1 codes: v[2j] in the low nibble of byte j, v[2j+1] in the
// high one (round to nearest even, saturating at 6)
__device__ __forceinline__ uint32_t e2m1x8_rn_satfinite(float v0, float v1, float v2, float v3, float v4, float v5,
                                                        float v6, float v7) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return out;
}

// per half of two packed bf16x2: max(|a|, |b|) with the sign bit set to sign(a) xor sign(b)
// (IEEE maxNum on the magnitudes: a NaN operand yields the other one); the caller clears the sign
__device__ __forceinline__ uint32_t bf16x2_max_abs(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// RN(p / 6) for float32 p, as Markstein's correction of the product by the rounded reciprocal for a
// divisor known in advance (Markstein, "IA-64 and Elementary Functions", 2000; Brisebarre, Muller
// and Raina, IEEE Trans. Computers 53(8), 2004): z = RN(1/6), q0 = RN(p z), r = p - 6 q0 (exact
// with an FMA), q1 = RN(q0 + r z).  Exact for every p whose quotient is a normal float32: the true
// quotient p/6 lies at least ulp/6 from every rounding midpoint (an fp32 p times 1/3 has no 25-bit
// expansion), while q0 + r z differs from it by at most |r| |z - 1/6| <= 9 ulp * 2^-27.  Checked
// exhaustively over all 2^23 significands on the host.  Quotients below the normal range all
// become E4M3 0 either way; an infinite or NaN p keeps q0 (inf or NaN, as the division gives).
__device__ __forceinline__ float div6_rn(float p) {
    const float z = 0x1.555556p-3f;                        // RN(1/6)
    const float q0 = __fmul_rn(p, z);
    const float r = __fmaf_rn(-q0, 6.0f, p);
    const float q1 = __fmaf_rn(r, z, q0);
    return fabsf(p) < INFINITY ? q1 : q0;
}

// {a.x * s, a.y * s}, each rounded to nearest even (one packed multiply)
__device__ __forceinline__ float2 mul2_rn(float2 a, float s) {
    uint64_t d;
    asm("{\n\t.reg .b64 pa, ps;\n\t"
        "mov.b64 pa, {%1, %2};\n\t"
        "mov.b64 ps, {%3, %3};\n\t"
        "mul.rn.f32x2 %0, pa, ps;\n\t}"
        : "=l"(d) : "f"(a.x), "f"(a.y), "f"(s));
    return make_float2(__uint_as_float((uint32_t)d), __uint_as_float((uint32_t)(d >> 32)));
}

// One 16-element block held as 8 words of bf16 pairs: scale byte and 16 codes (8 bytes).
// `inv_tab[s]` = gs / value(s) for the E4M3 bytes s = 1..126 (the positive finite scales).
__device__ __forceinline__ uint32_t quantize_block(const uint4 w0, const uint4 w1, float gs, const float* inv_tab,
                                                   uint2& packed_out) {
    const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    uint32_t m = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = bf16x2_max_abs(m, wv[i]);
    m &= 0x7FFF7FFFu;
    const float amax = fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
    const uint32_t sfb = e4m3_rn_satfinite(div6_rn(__fmul_rn(amax, gs)));
    uint32_t packed[2] = {0u, 0u};
    if (sfb - 1u < 126u) {                                   // value(sf) > 0
        const float inv = inv_tab[sfb];
        float y[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 v = mul2_rn(make_float2(__uint_as_float(wv[i] << 16), __uint_as_float(wv[i] & 0xFFFF0000u)), inv);
            y[2 * i] = v.x;
            y[2 * i + 1] = v.y;
        }
        packed[0] = e2m1x8_rn_satfinite(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
        packed[1] = e2m1x8_rn_satfinite(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
    }
    packed_out = make_uint2(packed[0], packed[1]);
    return sfb;
}

// One thread per 16-element block per step; launch bounds for 8 resident CTAs (64 warps) per SM,
// so that enough loads are in flight to cover the memory latency.
__global__ void __launch_bounds__(kQuantThreads, 8)
quantize_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t k, const float* __restrict__ gs_ptr,
                uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
    __shared__ float inv_tab[128];
    const float gs = *gs_ptr;
    if (threadIdx.x < 128) {
        const float v = e4m3_value(threadIdx.x);
        inv_tab[threadIdx.x] = v > 0.0f ? __fdiv_rn(gs, v) : 0.0f;
    }
    __syncthreads();
    const int64_t nb = k / 16;                               // blocks per row (a multiple of 4)
    const int64_t rows_p = (rows + 127) / 128 * 128;
    const int64_t total = rows_p * nb;                       // a multiple of 4
    const int64_t data = rows * nb;                          // blocks of the unpadded rows
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;  // a multiple of 32
    const int64_t stride_r = stride / nb, stride_c = stride % nb;
    const int lane = threadIdx.x & 31;
    int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
    int64_t r = (base + lane) / nb, c = (base + lane) % nb;  // this lane's block: row r, block c
    // every lane runs the same number of iterations, so the shuffles below see a full warp
    for (; base < total; base += stride) {
        const int64_t blk = base + lane;                     // = r * nb + c
        const bool live = blk < total;
        uint32_t sfb = 0;
        if (blk < data) {                                    // a row of the input (rows are contiguous)
            const uint4* src = reinterpret_cast<const uint4*>(x + blk * 16);
            uint2 packed;
            sfb = quantize_block(__ldg(src), __ldg(src + 1), gs, inv_tab, packed);
            *reinterpret_cast<uint2*>(codes + blk * 8) = packed;
        }
        // four consecutive blocks of a row: one 4-byte store into the swizzled scale atom
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, sfb, 1);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, sfb, 2);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, sfb, 3);
        if (live && (lane & 3) == 0) {
            const uint64_t ur = (uint64_t)r, uc = (uint64_t)c, unb = (uint64_t)nb;
            const uint64_t off = ((ur >> 7) * (unb >> 2) + (uc >> 2)) * 512 + (ur & 31) * 16 + ((ur >> 5) & 3) * 4;
            *reinterpret_cast<uint32_t*>(sf + off) = sfb | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
        c += stride_c;
        r += stride_r;
        if (c >= nb) {
            c -= nb;
            ++r;
        }
    }
}

}  // namespace nvfp4lora
