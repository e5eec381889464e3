// Persistent warp-specialised NVFP4 x NVFP4 GEMM with a fused BF16 LoRA term (sm_100a).
//
// Computes flashinfer.gemm.mm_nvfp4_lora's opening formula
//     out = bf16_rne(alpha * (dequant(a) @ dequant(b)^T) + lora_scale * (d @ lora_b^T) [+ bias])
// one 128 x BN output tile at a time, tiles strided over a persistent grid:
//   warp 0     TMA producer: A/B code tiles (2-D TMA, 128-byte swizzle) and the 512-byte scale
//              atoms (1-D bulk copies) per 256-wide K stage; after a tile's base stages, the
//              d / lora_b tiles of the LoRA term (64 ranks per stage).
//   warp 1     allocates TMEM; one thread issues tcgen05.cp (scale atoms -> TMEM) and the
//              block-scaled MMAs (kind::mxf4nvf4, 16-element UE4M3 scale vectors) into one of two
//              fp32 accumulators (tiles alternate), then the bf16 MMAs (kind::f16, K = r) of
//              the LoRA term: into a separate accumulator on the raw path ("Raw path" bullet),
//              into the tile's accumulator after the base product on the prepared path
//              ("Prepared path" bullet).
//   warps 2-5  epilogue: tcgen05.ld, release of the accumulator, v = alpha*acc
//              [; v = fma(s, lora_acc, v)] [; v += bias], one round-to-nearest-even to bf16,
//              then a 128B-swizzled shared-memory tile stored by TMA (or direct stores when
//              the row pitch of out is not a multiple of 16 bytes).
// With two accumulators the epilogue of tile i overlaps the MMAs of tile i+1.
// Zero-adapter path (Parameters: lora_scale): every role reads the LoRA scalar; when it equals 0
// no LoRA tile is loaded or multiplied and the epilogue is the adapter-off one, so the output is
// bitwise the adapter-off output.
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
    int tma_store;           // 1: out written through its tensor map (N % 8 == 0)
    int bias_vec;            // 1: bias rows may be read 16 bytes at a time (aligned, N % 8 == 0)
};

// Shared-memory plan of one CTA.  Each stage holds one A tile (128 rows x 128 bytes), one B
// tile (BN rows x 128 bytes) and their scale atoms; a LoRA stage reuses the A/B slots for a
// 128 x 64 bf16 d tile and a BN x 64 bf16 lora_b tile (also 128 bytes per row).  Two output
// staging tiles of 128 rows x 64 bf16 (128 bytes) feed the TMA stores.
template <int BN, int STAGES>
struct GemmSmem {
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int SFA_BYTES = 4 * 512;
    static constexpr int SFB_BYTES = (BN / 128) * 4 * 512;
    static constexpr int OUT_BYTES = 128 * 128;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int OUT_OFF = B_OFF + STAGES * B_BYTES;
    static constexpr int SFA_OFF = OUT_OFF + 2 * OUT_BYTES;
    static constexpr int SFB_OFF = SFA_OFF + STAGES * SFA_BYTES;
    static constexpr int BAR_OFF = SFB_OFF + STAGES * SFB_BYTES;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], lacc_empty, drain
    static constexpr int NUM_BARS = 2 * STAGES + 6;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int TOTAL = MISC_OFF + 16;
    static constexpr int DYN_BYTES = TOTAL + 1024;    // slack to align the base to 1024 bytes
};

// TMEM plan (columns of 32-bit cells, 128 lanes): two accumulators, the raw path's LoRA
// accumulator, then NSF scale slots used round-robin by the pipeline stages.  tcgen05.cp and
// tcgen05.mma issued by one thread execute in issue order, so a slot is never overwritten
// before the MMAs that read it; the round-robin keeps several stages of slack on top.
template <int BN, Mode MODE>
struct TmemPlan {
    static constexpr int ACC = 0;                     // accumulator b at ACC + b * BN
    static constexpr int LACC = 2 * BN;
    static constexpr int SF0 = (MODE == Mode::Raw) ? 3 * BN : 2 * BN;
    static constexpr int SFA_COLS = 4 * 4;            // 4 MMAs (K = 64 each) x 4 columns
    static constexpr int SFB_COLS = 4 * (BN / 32);    // 4 MMAs x BN/32 columns
    static constexpr int SLOT_COLS = SFA_COLS + SFB_COLS;
    static constexpr int NSF = (512 - SF0) / SLOT_COLS >= 4 ? 4 : (512 - SF0) / SLOT_COLS;
    static constexpr int USED = SF0 + NSF * SLOT_COLS;
    static constexpr int ALLOC = USED <= 256 ? 256 : 512;
    static_assert(NSF >= 1 && USED <= 512, "TMEM plan exceeds 512 columns");
};

constexpr int kGemmThreads = 192;
constexpr uint32_t kEpiBarrier = 1;     // named barrier of the 128 epilogue threads

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN, int STAGES, Mode MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_lb,
                  const __grid_constant__ CUtensorMap tm_out, const GemmArgs args) {
    using L = GemmSmem<BN, STAGES>;
    using T = TmemPlan<BN, MODE>;
    static_assert(BN == 128, "the epilogue and TMEM plan are written for BN = 128");
    constexpr uint32_t IDESC_F4 = idesc_nvf4(BN);
    constexpr uint32_t IDESC_BF16 = idesc_bf16(BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* empty = full + STAGES;
    uint64_t* tmem_full = empty + STAGES;      // [2]
    uint64_t* tmem_empty = tmem_full + 2;      // [2]
    uint64_t* lacc_empty = tmem_empty + 2;
    uint64_t* drain = lacc_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int lora_chunks_if_on = (args.r + 63) / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], 128);
        }
        mbar_init(lacc_empty, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tm_a);
        prefetch_tensor_map(&tm_b);
        if (MODE != Mode::Off) {
            prefetch_tensor_map(&tm_d);
            prefetch_tensor_map(&tm_lb);
        }
        if (args.tma_store) prefetch_tensor_map(&tm_out);
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
            float sv = 0.0f;
            if constexpr (MODE != Mode::Off) sv = *args.scale;   // consumed after the base stages
            int stage = 0;
            uint32_t phase = 0, filled = 0, filled_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
                const int m_blk = tile % args.m_tiles;
                const int n_blk = tile / args.m_tiles;
                const int items = args.k_stages + (sv != 0.0f ? lora_chunks_if_on : 0);
                for (int it = 0; it < items; ++it) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* sa = smem + L::A_OFF + stage * L::A_BYTES;
                    uint8_t* sb = smem + L::B_OFF + stage * L::B_BYTES;
                    if (it >= args.k_stages) {
                        const int c = it - args.k_stages;
                        mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
                        tma_load_2d(sa, &tm_d, &full[stage], c * 64, m_blk * 128);
                        tma_load_2d(sb, &tm_lb, &full[stage], c * 64, n_blk * BN);
                    } else {
                        int nsfb = 0;
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j)
                            nsfb += (n_blk * (BN / 128) + j < args.sf_row_blocks_b) ? 1 : 0;
                        mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES + 2048 + nsfb * 2048);
                        tma_load_2d(sa, &tm_a, &full[stage], it * 128, m_blk * 128);
                        tma_load_2d(sb, &tm_b, &full[stage], it * 128, n_blk * BN);
                        uint8_t* sfa = smem + L::SFA_OFF + stage * L::SFA_BYTES;
                        uint8_t* sfb = smem + L::SFB_OFF + stage * L::SFB_BYTES;
                        bulk_load(sfa, args.a_sf + ((size_t)m_blk * args.sf_atoms_k + it * 4) * 512, 2048,
                                  &full[stage]);
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j) {
                            const int rb = n_blk * (BN / 128) + j;
                            if (rb < args.sf_row_blocks_b)
                                bulk_load(sfb + j * 2048, args.b_sf + ((size_t)rb * args.sf_atoms_k + it * 4) * 512,
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
            float sv = 0.0f;
            if constexpr (MODE != Mode::Off) sv = *args.scale;
            int stage = 0, slot = 0;
            uint32_t phase = 0, lacc_uses = 0;
            bool ok = true;
            int i = 0;   // local tile counter
            for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x, ++i) {
                const int b = i & 1;
                const uint32_t acc_t = tmem + T::ACC + b * BN;
                if (!mbar_wait(&tmem_empty[b], ((i >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const bool lora_on = (MODE != Mode::Off) && sv != 0.0f;
                const int items = args.k_stages + (lora_on ? lora_chunks_if_on : 0);
                for (int it = 0; it < items; ++it) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                    const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                    if (it >= args.k_stages) {
                        const int c = it - args.k_stages;
                        if (MODE == Mode::Raw && c == 0) {
                            // the LoRA accumulator of the previous tile must have been read
                            if (!mbar_wait(lacc_empty, (lacc_uses & 1) ^ 1, abort_flag)) { ok = false; break; }
                            tc_fence_after();
                            ++lacc_uses;
                        }
                        const int rem = args.r - c * 64;
                        const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                        const uint32_t d_tmem = (MODE == Mode::Raw) ? tmem + T::LACC : acc_t;
                        for (int j = 0; j < ksteps; ++j) {
                            const uint32_t accum = (MODE == Mode::Raw) ? ((c > 0 || j > 0) ? 1u : 0u) : 1u;
                            tc_mma_bf16(d_tmem, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                        IDESC_BF16, accum);
                        }
                    } else {
                        const uint32_t sfa_t = tmem + T::SF0 + slot * T::SLOT_COLS;
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
                            tc_mma_nvf4(acc_t, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32), IDESC_F4,
                                        sfa_t + 4 * j, sfb_t + j * (BN / 32), (it > 0 || j > 0) ? 1u : 0u);
                        if (++slot == T::NSF) slot = 0;
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(&tmem_full[b]);
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
        const int rl = q * 32 + lane;                  // row within the tile
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const bool leader = (warp == 2 && lane == 0);  // issues the TMA stores
        float lora_s = 0.0f;
        if constexpr (MODE != Mode::Off) lora_s = *args.scale;
        const bool lora_on = (MODE != Mode::Off) && lora_s != 0.0f;
        const float alpha = *args.alpha;
        int chunk_ctr = 0;
        int i = 0;
        for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x, ++i) {
            const int b = i & 1;
            const int m_blk = tile % args.m_tiles;
            const int n_blk = tile / args.m_tiles;
            if (!mbar_wait(&tmem_full[b], (i >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const int row = m_blk * 128 + rl;
#pragma unroll 1
            for (int c = 0; c < BN / 64; ++c) {
                uint32_t acc[64];
                uint32_t lac[64];
                tmem_load_32(tmem + lane_off + T::ACC + b * BN + c * 64, *reinterpret_cast<uint32_t(*)[32]>(acc));
                tmem_load_32(tmem + lane_off + T::ACC + b * BN + c * 64 + 32,
                             *reinterpret_cast<uint32_t(*)[32]>(acc + 32));
                if (MODE == Mode::Raw && lora_on) {
                    tmem_load_32(tmem + lane_off + T::LACC + c * 64, *reinterpret_cast<uint32_t(*)[32]>(lac));
                    tmem_load_32(tmem + lane_off + T::LACC + c * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(lac + 32));
                }
                tmem_load_wait();
                if (c == BN / 64 - 1) {
                    // every column of this tile's accumulators is in registers: hand TMEM back
                    tc_fence_before();
                    mbar_arrive(&tmem_empty[b]);
                    if (MODE == Mode::Raw && lora_on) mbar_arrive(lacc_empty);
                }
                const int col0 = n_blk * BN + c * 64;
                float v[64];
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    float x = __fmul_rn(alpha, __uint_as_float(acc[k]));
                    if (MODE == Mode::Raw && lora_on) x = __fmaf_rn(lora_s, __uint_as_float(lac[k]), x);
                    v[k] = x;
                }
                if (args.bias != nullptr) {
                    if (args.bias_vec && col0 + 64 <= args.N) {
                        const uint4* bp = reinterpret_cast<const uint4*>(args.bias + col0);
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
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
                        for (int k = 0; k < 64; ++k)
                            if (col0 + k < args.N)
                                v[k] = __fadd_rn(v[k], __uint_as_float((uint32_t)__ldg(args.bias + col0 + k) << 16));
                    }
                }
                if (args.tma_store) {
                    // stage the 128 x 64 bf16 chunk in shared memory with the 128-byte swizzle
                    // (16-byte unit j of row r sits at unit j ^ (r % 8)) and store it with TMA
                    uint8_t* stile = smem + L::OUT_OFF + (chunk_ctr & 1) * L::OUT_BYTES;
                    if (leader) bulk_wait_group_read<1>();     // the store that used this buffer is done
                    named_barrier_sync(kEpiBarrier, 128);
                    uint8_t* srow = stile + rl * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 w = make_uint4(pack_bf16x2(v[j * 8 + 0], v[j * 8 + 1]),
                                                   pack_bf16x2(v[j * 8 + 2], v[j * 8 + 3]),
                                                   pack_bf16x2(v[j * 8 + 4], v[j * 8 + 5]),
                                                   pack_bf16x2(v[j * 8 + 6], v[j * 8 + 7]));
                        *reinterpret_cast<uint4*>(srow + ((j ^ (rl & 7)) << 4)) = w;
                    }
                    fence_proxy_async_smem();
                    named_barrier_sync(kEpiBarrier, 128);
                    if (leader) {
                        tma_store_2d(&tm_out, stile, col0, m_blk * 128);
                        bulk_commit_group();
                    }
                    ++chunk_ctr;
                } else if (row < args.M) {
                    uint16_t* orow = args.out + (size_t)row * args.N;
#pragma unroll
                    for (int k = 0; k < 64; ++k)
                        if (col0 + k < args.N) {
                            __nv_bfloat16 h = __float2bfloat16_rn(v[k]);
                            orow[col0 + k] = *reinterpret_cast<uint16_t*>(&h);
                        }
                }
            }
        }
        if (leader) bulk_wait_group_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, T::ALLOC);
    }
}

}  // namespace nvfp4lora
