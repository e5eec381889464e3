// SM-pair (cta_group::2) NVFP4 x NVFP4 GEMM with the folded LoRA term, for large M (sm_100a).
//
// Same operation as gemm.cuh (flashinfer.gemm.mm_nvfp4_lora, opening formula), for the adapter-
// off and prepared paths ("Prepared path" bullet: the folded LoRA term goes into the base
// accumulator after the base product, alpha is applied once).  A cluster of two CTAs computes
// one 256 x 256 output tile per step with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64):
//   * each CTA loads its own 128 rows of A and its half of the tile's 256 B rows (the leader the
//     first 128), at the same shared-memory offsets, plus its A scale atoms and the scale atoms
//     of all 256 B rows; the loads are cta_group::2 TMA copies whose bytes complete on the
//     leader's barrier, so each SM moves 38 KB per K stage instead of 54 KB for the same work;
//   * the leader's single MMA thread copies both CTAs' scale atoms into their TMEM
//     (tcgen05.cp.cta_group::2) and issues the MMAs and, on the prepared path, the bf16 LoRA MMAs
//     (kind::f16, N = 256) for both; stage releases and the tile hand-off are multicast commits
//     to both CTAs' barriers;
//   * each CTA drains its own 128 accumulator lanes (8 epilogue warps, 128 columns each), then
//     v = alpha*acc [+ bias], one RNE to bf16, TMA stores; its threads release the accumulator
//     on the leader's barrier (remote arrivals from the peer).
// The raw path keeps the single-SM kernel: its LoRA term needs a separate accumulator whose
// 128-column halves do not match the pair's split of N.  No multicast load is used.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace nvfp4lora {

constexpr int kPairTileM = 256;          // output rows per pair tile (128 per CTA)
constexpr int kPairStages = 4;

struct PairArgs {
    const float* alpha;
    const float* scale;      // Prepared: the fold's ratio; Off: unused
    const uint16_t* bias;    // bf16 [N] or null
    uint16_t* out;           // bf16 [M, N]
    int M, N, K, r;
    int m_pairs, n_tiles, num_tiles;   // pair tiles: m fastest
    int k_stages;            // K / 256
    int sf_atoms_k;          // K / 64
    int vec_out;             // rows of out (and bias) 16-byte aligned: TMA stores, bias in smem
};

template <int STAGES>
struct PairSmem {
    static constexpr int A_BYTES = 128 * 128;             // 128 rows x 128 bytes (256 codes)
    static constexpr int B_BYTES = 128 * 128;             // this CTA's half of the B tile
    static constexpr int SFA_BYTES = 4 * 512;             // 4 atoms: 128 rows x 4 K steps
    static constexpr int SFB_BYTES = 2 * 4 * 512;         // both 128-row blocks of the B tile
    static constexpr int STAGE_TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int LORA_TX = 128 * 128 + 128 * 128; // d rows + lora half, 64 ranks each
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int SFA_OFF = B_OFF + STAGES * B_BYTES;
    static constexpr int SFB_OFF = SFA_OFF + STAGES * SFA_BYTES;
    static constexpr int BIAS_BYTES = kTileN * 2;
    static constexpr int BIAS_OFF = SFB_OFF + STAGES * SFB_BYTES;
    static constexpr int OUT_BOX_BYTES = kOutBoxCols * kOutBoxRows * 2;
    static constexpr int OUT_OFF = BIAS_OFF + 2 * BIAS_BYTES;
    static constexpr int BAR_OFF = OUT_OFF + kEpiWarps * kOutBoxes * OUT_BOX_BYTES;
    // full[S], empty[S], tmem_full, acc_empty, drain, bias_full[2], bias_empty[2]
    static constexpr int NUM_BARS = 2 * STAGES + 7;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int TOTAL = MISC_OFF + 16;
    static constexpr int DYN_BYTES = TOTAL + 1024;
    static_assert(DYN_BYTES <= 232448, "pair shared-memory plan exceeds 227 KB");
};

// TMEM (same columns in both CTAs): the 256-column accumulator and NSF scale slots, used round-
// robin by the base stages.  Copies and MMAs come from one thread in issue order, so a slot is
// rewritten only after the MMAs that read it.
struct PairTmem {
    static constexpr int ACC = 0;
    static constexpr int SF0 = kTileN;
    static constexpr int SFA_COLS = 4 * 4;
    static constexpr int SFB_COLS = 4 * (kTileN / 32);
    static constexpr int SLOT_COLS = SFA_COLS + SFB_COLS;
    static constexpr int NSF = 5;
    static constexpr int ALLOC = 512;
    static_assert(SF0 + NSF * SLOT_COLS <= ALLOC, "pair TMEM plan exceeds 512 columns");
};

template <int STAGES, Mode MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                       const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_lb,
                       const __grid_constant__ CUtensorMap tm_out, const PairArgs args) {
    static_assert(MODE != Mode::Raw, "the raw path uses the single-SM kernel");
    using L = PairSmem<STAGES>;
    using T = PairTmem;
    constexpr uint32_t IDESC_F4 = idesc_nvf4_m(kPairTileM, kTileN);
    constexpr uint32_t IDESC_BF16 = idesc_bf16_m(kPairTileM, kTileN);
    constexpr uint16_t kBoth = 0x3;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);   // the leader's is used
    uint64_t* empty = full + STAGES;
    uint64_t* tmem_full = empty + STAGES;
    uint64_t* acc_empty = tmem_full + 1;                                // the leader's is used
    uint64_t* drain = acc_empty + 1;
    uint64_t* bias_full = drain + 1;
    uint64_t* bias_empty = bias_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();          // 0: the leader, which issues the MMAs
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int lora_chunks_if_on = (args.r + 63) / 64;

    if (threadIdx.x == 0) {
        prefetch_tensor_map(&tm_a);
        prefetch_tensor_map(&tm_b);
        prefetch_tensor_map(&tm_sfa);
        prefetch_tensor_map(&tm_sfb);
        if (args.vec_out) prefetch_tensor_map(&tm_out);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);          // the leader's expect_tx; bytes from both CTAs
            mbar_init(&empty[s], 1);         // the leader's multicast commit
        }
        mbar_init(tmem_full, 1);
        mbar_init(acc_empty, 2 * 32 * kEpiWarps);   // every epilogue thread of both CTAs
        mbar_init(drain, 1);
        for (int k = 0; k < 2; ++k) {
            mbar_init(&bias_full[k], 1);
            mbar_init(&bias_empty[k], 32 * kEpiWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, T::ALLOC);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // both CTAs' barriers exist before any copy completes on, or any thread arrives at, the peer
    cluster_arrive();
    cluster_wait();
    const uint32_t tmem = *tmem_slot;
    grid_launch_dependents();

    if (warp == 0) {
        // ------------------------------- TMA producer (both CTAs) -------------------------------
        if (lane == 0) {
            grid_dependency_wait();
            float sv = 0.0f;
            if constexpr (MODE == Mode::Prepared) sv = *args.scale;
            if (MODE == Mode::Prepared) {
                prefetch_tensor_map(&tm_d);
                prefetch_tensor_map(&tm_lb);
            }
            const bool lora_on = (MODE == Mode::Prepared) && sv != 0.0f;
            const bool bias_smem = args.bias != nullptr && args.vec_out;
            int stage = 0, tl = 0;
            uint32_t phase = 0, filled = 0, bias_issued = 0, bias_par = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < args.num_tiles; tile += npairs, ++tl) {
                const int m_pair = tile % args.m_pairs;
                const int n_blk = tile / args.m_pairs;
                const int row_a = m_pair * kPairTileM + (int)rank * 128;      // this CTA's A rows
                const int row_b = n_blk * kTileN + (int)rank * 128;           // this CTA's B half
                const int blk_a = m_pair * 2 + (int)rank;                     // its 128-row scale block
                if (bias_smem) {
                    const int bb = tl & 1;
                    if (!mbar_wait(&bias_empty[bb], ((tl >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    const int n0 = n_blk * kTileN;
                    const uint32_t bytes = (uint32_t)min(kTileN, args.N - n0) * 2u;   // N % 8 == 0
                    mbar_arrive_expect_tx(&bias_full[bb], bytes);
                    bulk_load(smem + L::BIAS_OFF + bb * L::BIAS_BYTES, args.bias + n0, bytes, &bias_full[bb]);
                    bias_issued |= 1u << bb;
                    bias_par = (bias_par & ~(1u << bb)) | ((((uint32_t)tl >> 1) & 1u) << bb);
                }
                const int items = args.k_stages + (lora_on ? lora_chunks_if_on : 0);
                for (int it = 0; it < items; ++it) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t lead_full = map_to_rank(smem_u32(&full[stage]), 0);
                    uint8_t* sa = smem + L::A_OFF + stage * L::A_BYTES;
                    uint8_t* sb = smem + L::B_OFF + stage * L::B_BYTES;
                    if (it < args.k_stages) {
                        if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * L::STAGE_TX);
                        tma_load_2d_pair(sa, &tm_a, lead_full, it * 128, row_a);
                        tma_load_2d_pair(sb, &tm_b, lead_full, it * 128, row_b);
                        // scale atoms through a [bytes / 128, 128] view: 16 rows = 4 atoms (2 KB)
                        tma_load_2d_pair(smem + L::SFA_OFF + stage * L::SFA_BYTES, &tm_sfa, lead_full, 0,
                                         (blk_a * args.sf_atoms_k + it * 4) * 4);
                        uint8_t* sfb = smem + L::SFB_OFF + stage * L::SFB_BYTES;
                        tma_load_2d_pair(sfb, &tm_sfb, lead_full, 0, ((n_blk * 2) * args.sf_atoms_k + it * 4) * 4);
                        tma_load_2d_pair(sfb + 2048, &tm_sfb, lead_full, 0,
                                         ((n_blk * 2 + 1) * args.sf_atoms_k + it * 4) * 4);
                    } else {
                        const int c = it - args.k_stages;
                        if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * L::LORA_TX);
                        tma_load_2d_pair(sa, &tm_d, lead_full, c * 64, row_a);
                        tma_load_2d_pair(sb, &tm_lb, lead_full, c * 64, row_b);
                    }
                    filled |= 1u << stage;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok || *abort_flag) {
                // Let this CTA's own copies land before it can exit (the pair's loads complete on
                // the leader's barriers; both CTAs meet at the final cluster barrier).
                for (int k = 0; k < 2; ++k)
                    if ((bias_issued >> k) & 1u) mbar_wait(&bias_full[k], (bias_par >> k) & 1u, nullptr);
            }
            (void)filled;
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer (the leader) -------------------------------
        if (lane == 0 && rank == 0) {
            grid_dependency_wait();
            float sv = 0.0f;
            if constexpr (MODE == Mode::Prepared) sv = *args.scale;
            const bool lora_on = (MODE == Mode::Prepared) && sv != 0.0f;
            int stage = 0, slot = 0;
            uint32_t phase = 0;
            bool ok = true;
            int i = 0;
            for (int tile = pair; ok && tile < args.num_tiles; tile += npairs, ++i) {
                // both CTAs' epilogues have read the previous tile's accumulator
                if (!mbar_wait_cluster(acc_empty, (i & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int it = 0; ok && it < args.k_stages; ++it) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                    const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                    const uint32_t sfa_t = tmem + T::SF0 + slot * T::SLOT_COLS;
                    const uint32_t sfb_t = sfa_t + T::SFA_COLS;
                    const uint32_t sfa_s = smem_u32(smem + L::SFA_OFF + stage * L::SFA_BYTES);
                    const uint32_t sfb_s = smem_u32(smem + L::SFB_OFF + stage * L::SFB_BYTES);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        tc_copy_scale_atom_pair(sfa_t + 4 * j, sdesc_scale_atom(sfa_s + j * 512));
                        tc_copy_scale_atom_pair(sfb_t + 8 * j, sdesc_scale_atom(sfb_s + j * 512));
                        tc_copy_scale_atom_pair(sfb_t + 8 * j + 4, sdesc_scale_atom(sfb_s + 2048 + j * 512));
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc_mma_nvf4_pair(tmem + T::ACC, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                         IDESC_F4, sfa_t + 4 * j, sfb_t + 8 * j, (it > 0 || j > 0) ? 1u : 0u);
                    tc_commit_pair_multicast(&empty[stage], kBoth);
                    if (++slot == T::NSF) slot = 0;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                if (lora_on) {
                    // the folded LoRA term into the same accumulator, after the base product
                    for (int c = 0; ok && c < lora_chunks_if_on; ++c) {
                        if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                        const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                        const int rem = args.r - c * 64;
                        const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                        for (int j = 0; j < ksteps; ++j)
                            tc_mma_bf16_pair(tmem + T::ACC, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                             IDESC_BF16, 1u);
                        tc_commit_pair_multicast(&empty[stage], kBoth);
                        if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    }
                    if (!ok) break;
                }
                tc_commit_pair_multicast(tmem_full, kBoth);     // both CTAs' accumulators are complete
            }
            if (!ok || *abort_flag) {
                // Wait for the MMAs already issued before TMEM is released.
                tc_commit_pair_multicast(drain, 0x1);
                mbar_wait(drain, 0, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------- epilogue (both CTAs) -------------------------------
        const int q = warp & 3;                        // TMEM lane quarter of this warp
        const int h = (warp - 2) >> 2;                 // which 128 of the 256 columns
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        grid_dependency_wait();
        const float alpha = *args.alpha;
        const uint32_t lead_acc_empty = map_to_rank(smem_u32(acc_empty), 0);
        int i = 0, out_box = 0;
        for (int tile = pair; tile < args.num_tiles; tile += npairs, ++i) {
            const int m_pair = tile % args.m_pairs;
            const int n_blk = tile / args.m_pairs;
            if (!__all_sync(0xffffffffu, mbar_wait(tmem_full, i & 1, abort_flag))) break;
            tc_fence_after();
            uint32_t raw[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_load_32(tmem + lane_off + T::ACC + h * 128 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(raw + c * 32));
            tmem_load_wait();
            tc_fence_before();
            // the leader may start the next tile's MMAs once both CTAs hold their accumulators
            if (rank == 0) mbar_arrive(acc_empty);
            else mbar_arrive_remote(lead_acc_empty);
            float v[128];
#pragma unroll
            for (int k = 0; k < 128; ++k) v[k] = __fmul_rn(alpha, __uint_as_float(raw[k]));
            const int row0 = m_pair * kPairTileM + (int)rank * 128 + q * 32;   // this warp's 32 rows
            const int row = row0 + lane;
            const int col0 = n_blk * kTileN + h * 128;
            if (args.bias != nullptr) {
                if (args.vec_out) {
                    if (!mbar_wait(&bias_full[i & 1], (i >> 1) & 1, abort_flag)) break;
                    const uint4* bp =
                        reinterpret_cast<const uint4*>(smem + L::BIAS_OFF + (i & 1) * L::BIAS_BYTES) + h * 16;
#pragma unroll
                    for (int g8 = 0; g8 < 16; ++g8) {
                        const uint4 w = bp[g8];
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            v[g8 * 8 + 2 * e] = __fadd_rn(v[g8 * 8 + 2 * e], __uint_as_float(ws[e] << 16));
                            v[g8 * 8 + 2 * e + 1] = __fadd_rn(v[g8 * 8 + 2 * e + 1], __uint_as_float(ws[e] & 0xFFFF0000u));
                        }
                    }
                    mbar_arrive(&bias_empty[i & 1]);
                } else {
#pragma unroll
                    for (int k = 0; k < 128; ++k)
                        if (col0 + k < args.N)
                            v[k] = __fadd_rn(v[k], __uint_as_float((uint32_t)__ldg(args.bias + col0 + k) << 16));
                }
            }
            if (args.vec_out) {
                uint8_t* box0 = smem + L::OUT_OFF + (warp - 2) * kOutBoxes * L::OUT_BOX_BYTES;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint8_t* box = box0 + out_box * L::OUT_BOX_BYTES;
                    if (++out_box == kOutBoxes) out_box = 0;
                    if (lane == 0) bulk_wait_group_read<kOutBoxes - 1>();   // its previous store has read it
                    __syncwarp();
                    uint4* dst = reinterpret_cast<uint4*>(box + lane * 64);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int b8 = c * 32 + k * 8;
                        dst[k] = make_uint4(pack_bf16x2(v[b8], v[b8 + 1]), pack_bf16x2(v[b8 + 2], v[b8 + 3]),
                                            pack_bf16x2(v[b8 + 4], v[b8 + 5]), pack_bf16x2(v[b8 + 6], v[b8 + 7]));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    const int x = col0 + c * kOutBoxCols;
                    if (lane == 0 && x < args.N && row0 < args.M) {
                        tma_store_2d(&tm_out, box, x, row0);
                        bulk_commit_group();
                    }
                }
            } else if (row < args.M) {
                uint16_t* orow = args.out + (size_t)row * args.N + col0;
#pragma unroll
                for (int k = 0; k < 128; ++k)
                    if (col0 + k < args.N) {
                        __nv_bfloat16 hv = __float2bfloat16_rn(v[k]);
                        orow[k] = *reinterpret_cast<uint16_t*>(&hv);
                    }
            }
        }
        if (args.vec_out && lane == 0) bulk_wait_group_all();
    }

    // Neither CTA leaves (or gives TMEM back) while the other may still reach its barriers or the
    // leader's MMAs its TMEM: the whole pair meets here first.
    tc_fence_before();
    __syncthreads();
    cluster_arrive();
    cluster_wait();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, T::ALLOC);
    }
}

}  // namespace nvfp4lora
