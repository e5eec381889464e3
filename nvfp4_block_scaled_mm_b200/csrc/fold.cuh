// The LoRA fold (flashinfer.gemm.prepare_nvfp4_lora_adapter, summary paragraph):
//     ratio       = div.rn.f32(fp32(lora_scale), fp32(alpha[0]))
//     b_folded[i] = bf16_rne(fp32(lora_b[i]) * ratio)
// Both the eager prepare and the in-place refold launch this kernel, so the two are bitwise
// equal by construction.  The ratio is computed on the device (no host read) and stored in
// the adapter's device scalar, where the prepared GEMM reads it for the zero-adapter test.
// HBM-bound: 2 bytes read + 2 bytes written per element, 16 bytes per thread per access.
#pragma once

#include <cstdint>

namespace nvfp4lora {

// float32 -> bf16 bits, round to nearest, ties to even; every NaN becomes 0x7FC0.
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float x) {
    const uint32_t u = __float_as_uint(x);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0x7FC0u;
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

__device__ __forceinline__ uint32_t fold_pair(uint32_t two, float ratio) {
    const float lo = __fmul_rn(__uint_as_float(two << 16), ratio);
    const float hi = __fmul_rn(__uint_as_float(two & 0xFFFF0000u), ratio);
    return f32_to_bf16_bits(lo) | (f32_to_bf16_bits(hi) << 16);
}

constexpr int kFoldThreads = 256;

// `groups` = N*r/8 (r % 8 == 0): each thread folds 8 bf16 values (one 16-byte load/store).
__global__ void __launch_bounds__(kFoldThreads)
fold_kernel(const uint16_t* lora_b, const float* lora_scale, const float* alpha,
            uint16_t* b_folded, float* ratio_out, int64_t groups) {
    // Launched with programmatic dependent launch: the CTAs start while the previous kernel on
    // the stream (typically the GEMM that reads b_folded) finishes, and wait for it here before
    // any read or write.  A dependent GEMM may begin its prologue at once; it still waits for
    // this grid before reading.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const float ratio = __fdiv_rn(*lora_scale, *alpha);
    if (blockIdx.x == 0 && threadIdx.x == 0) *ratio_out = ratio;
    const uint4* src = reinterpret_cast<const uint4*>(lora_b);
    uint4* dst = reinterpret_cast<uint4*>(b_folded);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < groups;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 w = src[i];
        dst[i] = make_uint4(fold_pair(w.x, ratio), fold_pair(w.y, ratio), fold_pair(w.z, ratio),
                            fold_pair(w.w, ratio));
    }
}

}  // namespace nvfp4lora
