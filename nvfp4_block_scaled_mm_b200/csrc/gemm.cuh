// Persistent warp-specialised NVFP4 x NVFP4 GEMM with a fused BF16 LoRA term (sm_100a).
//
// Computes flashinfer.gemm.mm_nvfp4_lora's opening formula
//     out = bf16_rne(alpha * (dequant(a) @ dequant(b)^T) + lora_scale * (d @ lora_b^T) [+ bias])
// for one 128 x BN output tile at a time:
//   warp 0     TMA producer: A/B code tiles (2-D TMA, 128-byte swizzle), the 512-byte scale
//              atoms (1-D bulk copies), and for the LoRA term the d / lora_b tiles.
//   warp 1     allocates TMEM; one thread issues tcgen05.cp (scales -> TMEM) and the
//              block-scaled MMAs (kind::mxf4nvf4, 16-element UE4M3 scale vectors) into an
//              fp32 accumulator, plus the bf16 MMAs (kind::f16, K = r) of the LoRA term:
//              into its own accumulator on the raw path ("Raw path" bullet), into the base
//              accumulator after the base product on the prepared path ("Prepared path").
//   warps 2-5  epilogue: tcgen05.ld, v = alpha*acc [; v = fma(s, lora_acc, v)] [; v += bias],
//              one round-to-nearest-even to bf16, store.
// Zero-adapter path (Parameters: lora_scale): every thread reads the LoRA scalar once; when
// it equals 0 no LoRA tile is loaded or multiplied and the epilogue is the adapter-off one,
// so the output is bitwise the adapter-off output.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace nvfp4lora {

enum class Mode : int { Off = 0, Raw = 1, Prepared = 2 };

struct GemmArgs {
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const float* alpha;
    const float* scale;      // Raw: lora_scale; Prepared: the fold's ratio; Off: unused
    const uint16_t* bias;    // bf16 [N] or null
    uint16_t* out;           // bf16 [M, N]
    int M, N, K, r;
    int m_tiles, n_tiles, num_tiles;
    int k_stages;            // K / 256: one pipeline stage = 256 K-elements = 128 bytes per row
    int sf_atoms_k;          // K / 64: 512-byte scale atoms per 128-row block
    int sf_row_blocks_b;     // ceil(N / 128): 128-row scale blocks present in b_sf
};

// Shared-memory plan of one CTA.  Each stage holds one A tile (128 rows x 128 bytes), one B
// tile (BN rows x 128 bytes) and their scale atoms; a LoRA stage reuses the A/B slots for a
// 128 x 64 bf16 d tile and a BN x 64 bf16 lora_b tile (also 128 bytes per row).
template <int BN, int STAGES>
struct GemmSmem {
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int SFA_BYTES = 4 * 512;
    static constexpr int SFB_BYTES = (BN / 128) * 4 * 512;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int SFA_OFF = B_OFF + STAGES * B_BYTES;
    static constexpr int SFB_OFF = SFA_OFF + STAGES * SFA_BYTES;
    static constexpr int BAR_OFF = SFB_OFF + STAGES * SFB_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 3;   // full, empty, tmem_full, tmem_empty, drain
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int TOTAL = MISC_OFF + 16;
    static constexpr int DYN_BYTES = TOTAL + 1024;    // slack to align the base to 1024 bytes
};

// TMEM plan (columns of 32-bit cells, 128 lanes): the accumulator, the raw path's LoRA
// accumulator, then one scale region per pipeline stage.  A stage's region is rewritten only
// after the MMAs that read it have completed (the producer waits for their commit before
// refilling the stage whose copy lands there).
template <int BN, int STAGES, Mode MODE>
struct TmemPlan {
    static constexpr int ACC = 0;
    static constexpr int LACC = BN;
    static constexpr int SF0 = (MODE == Mode::Raw) ? 2 * BN : BN;
    static constexpr int SFA_COLS = 4 * 4;            // 4 MMAs (K = 64 each) x 4 columns
    static constexpr int SFB_COLS = 4 * (BN / 32);    // 4 MMAs x BN/32 columns
    static constexpr int STAGE_COLS = SFA_COLS + SFB_COLS;
    static constexpr int USED = SF0 + STAGES * STAGE_COLS;
    static constexpr int ALLOC = USED <= 32 ? 32 : USED <= 64 ? 64 : USED <= 128 ? 128
                               : USED <= 256 ? 256 : 512;
    static_assert(USED <= 512, "TMEM plan exceeds 512 columns");
};

constexpr int kGemmThreads = 192;

// Position `it` of a tile's stage sequence: a LoRA chunk (64 ranks) or a base K-stage.
__device__ __forceinline__ void tile_item(int it, int k_stages, int lora_chunks, bool lora_first,
                                          bool& is_lora, int& idx) {
    if (lora_first) {
        is_lora = it < lora_chunks;
        idx = is_lora ? it : it - lora_chunks;
    } else {
        is_lora = it >= k_stages;
        idx = is_lora ? it - k_stages : it;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN, int STAGES, Mode MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_lb,
                  const GemmArgs args) {
    using L = GemmSmem<BN, STAGES>;
    using T = TmemPlan<BN, STAGES, MODE>;
    static_assert(BN % 128 == 0 && BN <= 256, "BN must be 128 or 256");
    constexpr uint32_t IDESC_F4 = idesc_nvf4(BN);
    constexpr uint32_t IDESC_BF16 = idesc_bf16(BN);
    constexpr bool kLoraFirst = (MODE == Mode::Raw);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* empty = full + STAGES;
    uint64_t* tmem_full = empty + STAGES;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* drain = tmem_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // The zero-adapter decision, taken identically by every thread.
    float lora_s = 0.0f;
    bool lora_on = false;
    if constexpr (MODE != Mode::Off) {
        lora_s = *args.scale;
        lora_on = (lora_s != 0.0f);
    }
    const int lora_chunks = lora_on ? (args.r + 63) / 64 : 0;
    const int items = args.k_stages + lora_chunks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tm_a);
        prefetch_tensor_map(&tm_b);
        if (lora_on) {
            prefetch_tensor_map(&tm_d);
            prefetch_tensor_map(&tm_lb);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, T::ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, filled = 0, filled_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
                const int m_blk = tile % args.m_tiles;
                const int n_blk = tile / args.m_tiles;
                for (int it = 0; it < items; ++it) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    bool is_lora; int idx;
                    tile_item(it, args.k_stages, lora_chunks, kLoraFirst, is_lora, idx);
                    uint8_t* sa = smem + L::A_OFF + stage * L::A_BYTES;
                    uint8_t* sb = smem + L::B_OFF + stage * L::B_BYTES;
                    if (is_lora) {
                        mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
                        tma_load_2d(sa, &tm_d, &full[stage], idx * 64, m_blk * 128);
                        tma_load_2d(sb, &tm_lb, &full[stage], idx * 64, n_blk * BN);
                    } else {
                        int nsfb = 0;
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j)
                            nsfb += (n_blk * (BN / 128) + j < args.sf_row_blocks_b) ? 1 : 0;
                        mbar_arrive_expect_tx(&full[stage],
                                              L::A_BYTES + L::B_BYTES + 2048 + nsfb * 2048);
                        tma_load_2d(sa, &tm_a, &full[stage], idx * 128, m_blk * 128);
                        tma_load_2d(sb, &tm_b, &full[stage], idx * 128, n_blk * BN);
                        uint8_t* sfa = smem + L::SFA_OFF + stage * L::SFA_BYTES;
                        uint8_t* sfb = smem + L::SFB_OFF + stage * L::SFB_BYTES;
                        bulk_load(sfa, args.a_sf + ((size_t)m_blk * args.sf_atoms_k + idx * 4) * 512,
                                  2048, &full[stage]);
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j) {
                            const int rb = n_blk * (BN / 128) + j;
                            if (rb < args.sf_row_blocks_b)
                                bulk_load(sfb + j * 2048,
                                          args.b_sf + ((size_t)rb * args.sf_atoms_k + idx * 4) * 512,
                                          2048, &full[stage]);
                        }
                    }
                    filled |= 1u << stage;
                    filled_parity = (filled_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok || *abort_flag) {
                // Let every copy already issued land before the CTA can exit.
                for (int s = 0; s < STAGES; ++s)
                    if ((filled >> s) & 1u) mbar_wait(&full[s], (filled_parity >> s) & 1u, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, tphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
                if (!mbar_wait(tmem_empty, tphase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int it = 0; it < items; ++it) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    bool is_lora; int idx;
                    tile_item(it, args.k_stages, lora_chunks, kLoraFirst, is_lora, idx);
                    const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                    const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                    if (is_lora) {
                        const int rem = args.r - idx * 64;
                        const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                        const uint32_t d_tmem = tmem + (MODE == Mode::Raw ? T::LACC : T::ACC);
                        for (int j = 0; j < ksteps; ++j) {
                            const uint32_t acc = (MODE == Mode::Raw) ? ((idx > 0 || j > 0) ? 1u : 0u) : 1u;
                            tc_mma_bf16(d_tmem, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                        IDESC_BF16, acc);
                        }
                    } else {
                        const uint32_t sfa_t = tmem + T::SF0 + stage * T::STAGE_COLS;
                        const uint32_t sfb_t = sfa_t + T::SFA_COLS;
                        const uint32_t sfa_s = smem_u32(smem + L::SFA_OFF + stage * L::SFA_BYTES);
                        const uint32_t sfb_s = smem_u32(smem + L::SFB_OFF + stage * L::SFB_BYTES);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc_copy_scale_atom(sfa_t + 4 * j, sdesc_scale_atom(sfa_s + j * 512));
#pragma unroll
                        for (int jb = 0; jb < BN / 128; ++jb)
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                tc_copy_scale_atom(sfb_t + j * (BN / 32) + 4 * jb,
                                                   sdesc_scale_atom(sfb_s + jb * 2048 + j * 512));
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc_mma_nvf4(tmem + T::ACC, sdesc_sw128(a_addr + j * 32),
                                        sdesc_sw128(b_addr + j * 32), IDESC_F4, sfa_t + 4 * j,
                                        sfb_t + j * (BN / 32), (idx > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(tmem_full);
                tphase ^= 1;
            }
            if (!ok || *abort_flag) {
                // Wait for the MMAs already issued before TMEM is released.
                tc_commit(drain);
                mbar_wait(drain, 0, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------- epilogue -----------------------------------
        const int q = warp & 3;                        // TMEM lane quarter of this warp
        const float alpha = *args.alpha;
        const bool vec_ok = (args.N % 8) == 0;
        uint32_t tphase = 0;
        for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x) {
            const int m_blk = tile % args.m_tiles;
            const int n_blk = tile / args.m_tiles;
            if (!mbar_wait(tmem_full, tphase, abort_flag)) break;
            tc_fence_after();
            const int row = m_blk * 128 + q * 32 + lane;
            const uint32_t lane_off = (uint32_t)(q * 32) << 16;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t acc[32];
                uint32_t lac[32];
                tmem_load_32(tmem + lane_off + T::ACC + c * 32, acc);
                if (MODE == Mode::Raw && lora_on) tmem_load_32(tmem + lane_off + T::LACC + c * 32, lac);
                tmem_load_wait();
                const int col0 = n_blk * BN + c * 32;
                const bool full_chunk = vec_ok && (col0 + 32 <= args.N);
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float x = __fmul_rn(alpha, __uint_as_float(acc[i]));
                    if (MODE == Mode::Raw && lora_on) x = __fmaf_rn(lora_s, __uint_as_float(lac[i]), x);
                    v[i] = x;
                }
                if (args.bias != nullptr) {
                    if (full_chunk) {
                        const uint4* bp = reinterpret_cast<const uint4*>(args.bias + col0);
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const uint4 w = __ldg(bp + g);
                            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                v[g * 8 + 2 * h] = __fadd_rn(v[g * 8 + 2 * h], __uint_as_float(ws[h] << 16));
                                v[g * 8 + 2 * h + 1] =
                                    __fadd_rn(v[g * 8 + 2 * h + 1], __uint_as_float(ws[h] & 0xFFFF0000u));
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (col0 + i < args.N)
                                v[i] = __fadd_rn(v[i], __uint_as_float((uint32_t)__ldg(args.bias + col0 + i) << 16));
                    }
                }
                if (row < args.M) {
                    uint16_t* orow = args.out + (size_t)row * args.N;
                    if (full_chunk) {
                        uint4* op = reinterpret_cast<uint4*>(orow + col0);
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            op[g] = make_uint4(pack_bf16x2(v[g * 8 + 0], v[g * 8 + 1]),
                                               pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]),
                                               pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]),
                                               pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (col0 + i < args.N) {
                                __nv_bfloat16 h = __float2bfloat16_rn(v[i]);
                                orow[col0 + i] = *reinterpret_cast<uint16_t*>(&h);
                            }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tmem_empty);
            tphase ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, T::ALLOC);
    }
}

}  // namespace nvfp4lora
