// SM-pair (cta_group::2) NVFP4 x NVFP4 GEMM with the folded LoRA term, for large M (sm_100a).
//
// Same operation as gemm.cuh (flashinfer.gemm.mm_nvfp4_lora, opening formula), for the adapter-
// off and prepared paths ("Prepared path" bullet: the folded LoRA term goes into the base
// accumulator after the base product, alpha is applied once).  A cluster of two CTAs computes
// one 256 x 256 output tile per step with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64):
//   * each CTA loads its own 128 rows of A and its half of the tile's 256 B rows (the leader the
//     first 128), at the same shared-memory offsets, with cta_group::2 TMA copies whose bytes
//     complete on the leader's barrier, so each SM moves 32 KB of codes per K stage instead of
//     48 KB for the same work;
//   * a second producer thread per CTA bulk-copies its A scale atoms and the scale atoms of all
//     256 B rows into a ring of its own, which the staging warps recycle as soon as they have
//     read it, so the scales of a stage arrive several stages ahead of its MMAs;
//   * four staging warps per CTA (one per TMEM lane quarter) write the stage's scale atoms from
//     shared memory into a TMEM scale slot with tcgen05.st, in the layout a 32x128b.warpx4 copy
//     gives, and report to the leader.  A scale copy (tcgen05.cp) shares the tensor pipe with
//     the MMAs; a register store does not, so the MMAs run back to back;
//   * the leader's single MMA thread issues the block-scaled MMAs and, on the prepared path, the
//     bf16 LoRA MMAs (kind::f16, N = 256) for both CTAs; stage, slot and accumulator hand-offs
//     are multicast commits to both CTAs' barriers;
//   * each CTA drains its own 128 accumulator lanes (8 epilogue warps, 128 columns each), then
//     v = alpha*acc [+ bias], one RNE to bf16, TMA stores; its threads release the accumulator
//     on the leader's barrier (remote arrivals from the peer).
// Raw path ("Raw path" bullet: alpha and lora_scale stay independent): the LoRA term goes into a
// separate 128-column accumulator, one N-half at a time (M = 256, N = 128 per instruction, each
// CTA holding 64 of the half's lora_b rows); the epilogue warps of the first half read it and
// release it before the second half is issued.
// Registers are split by warpgroup (setmaxnreg): producer/MMA and staging warps give theirs to
// the epilogue warpgroups.  No multicast load is used.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace nvfp4lora {

constexpr int kPairTileM = 256;          // output rows per pair tile (128 per CTA)
// Code-tile stages: 5 x 32 KB in flight per SM.  The room comes from the epilogue's output
// staging, one 32 x 32 box per warp (each box is rewritten once its previous store has read it;
// the epilogue has ample slack).  Against 4 stages with 3 boxes per warp: raw 4096^3 44.7 ->
// 43.3 us, raw 2048 x 28672 x 8192 261 -> 254 us, prepared 246 -> 239 us, adapter-off level.
constexpr int kPairStages = 5;
constexpr int kPairOutBoxes = 1;
constexpr int kPairSfStages = 4;         // scale-atom ring (own barriers, recycled by staging)
constexpr int kPairThreads = 512;
// Raw path: a tile's second LoRA half is issued this many base stages into the next tile, so that
// the epilogue warps have read the first half by then.
constexpr int kRawHalf1At = 4;        // 4 warpgroups: producer/MMA, staging, 2 x epilogue
// Registers per thread after the split.  The block is launched with 512 x 128; the split must not
// exceed that pool (setmaxnreg.inc waits for registers that the other warpgroups give back).
constexpr int kPairRegsLaunch = 128;
constexpr int kPairRegsCtl = 80;         // warpgroup 0: producers, MMA issuer, one idle warp
constexpr int kPairRegsStage = 72;       // warpgroup 1: scale staging
constexpr int kPairRegsEpi = 176;        // warpgroups 2 and 3: epilogue
static_assert(128 * (kPairRegsCtl + kPairRegsStage) + 256 * kPairRegsEpi <= kPairThreads * kPairRegsLaunch,
              "pair register split exceeds the launch's register pool");

struct PairArgs {
    const float* alpha;
    const float* scale;      // Prepared: the fold's ratio; Off: unused
    const uint8_t* a_sf;     // 128x4-swizzled scale atoms of a
    const uint8_t* b_sf;     // and of b
    const uint16_t* bias;    // bf16 [N] or null
    uint16_t* out;           // bf16 [M, N]
    int M, N, K, r;
    int m_pairs, n_tiles, num_tiles;   // pair tiles: m fastest
    int k_stages;            // K / 256
    int sf_atoms_k;          // K / 64
    int sf_row_blocks_a;     // ceil(M / 128)
    int sf_row_blocks_b;     // ceil(N / 128)
    int vec_out;             // rows of out (and bias) 16-byte aligned: TMA stores, bias in smem
};

template <int STAGES>
struct PairSmem {
    static constexpr int A_BYTES = 128 * 128;             // 128 rows x 128 bytes (256 codes)
    static constexpr int B_BYTES = 128 * 128;             // this CTA's half of the B tile
    static constexpr int SFA_BYTES = 4 * 512;             // 4 atoms: 128 rows x 4 K steps
    static constexpr int SFB_BYTES = 2 * 4 * 512;         // both 128-row blocks of the B tile
    static constexpr int STAGE_TX = A_BYTES + B_BYTES;    // per CTA, on the leader's barrier
    static constexpr int LORA_TX = 128 * 128 + 128 * 128; // d rows + lora half, 64 ranks each
    static constexpr int LORA_HALF_TX = 128 * 128 + 64 * 128;  // raw: d rows + 64 lora rows of an N-half
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int SFA_OFF = B_OFF + STAGES * B_BYTES;
    static constexpr int SFB_OFF = SFA_OFF + kPairSfStages * SFA_BYTES;
    static constexpr int BIAS_BYTES = kTileN * 2;
    static constexpr int BIAS_OFF = SFB_OFF + kPairSfStages * SFB_BYTES;
    static constexpr int OUT_BOX_BYTES = kOutBoxCols * kOutBoxRows * 2;
    static constexpr int OUT_OFF = BIAS_OFF + 2 * BIAS_BYTES;
    static constexpr int BAR_OFF = OUT_OFF + kEpiWarps * kPairOutBoxes * OUT_BOX_BYTES;
    static constexpr int MAX_SLOTS = 8;
    // full[S], empty[S], sf_full[SF], sf_empty[SF], sf_ready[8], slot_free[8], tmem_full,
    // acc_empty, lacc_full, lacc_empty, drain, bias_full[2], bias_empty[2]
    static constexpr int NUM_BARS = 2 * STAGES + 2 * kPairSfStages + 2 * MAX_SLOTS + 9;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int TOTAL = MISC_OFF + 16;
    static constexpr int DYN_BYTES = TOTAL + 1024;
    static_assert(DYN_BYTES <= 232448, "pair shared-memory plan exceeds 227 KB");
};

// TMEM (same columns in both CTAs): the 256-column accumulator, NSF scale slots used round-robin
// by the base stages, and on the raw path the 128-column LoRA accumulator.  A slot is restaged
// only after the commit that follows the MMAs of its previous stage (slot_free).
template <Mode MODE>
struct PairTmem {
    static constexpr int ACC = 0;
    static constexpr int SF0 = kTileN;
    static constexpr int SFA_COLS = 4 * 4;
    static constexpr int SFB_COLS = 4 * (kTileN / 32);
    static constexpr int SLOT_COLS = SFA_COLS + SFB_COLS;
    static constexpr int NSF = (MODE == Mode::Raw) ? 2 : 5;
    static constexpr int LACC = SF0 + NSF * SLOT_COLS;
    static constexpr int USED = (MODE == Mode::Raw) ? LACC + 128 : LACC;
    static constexpr int ALLOC = 512;
    static_assert(USED <= ALLOC, "pair TMEM plan exceeds 512 columns");
    static_assert(NSF <= PairSmem<kPairStages>::MAX_SLOTS, "too many scale slots for the barriers");
};

template <int STAGES, Mode MODE>
__global__ void __launch_bounds__(kPairThreads, 1)
nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_lb,
                       const __grid_constant__ CUtensorMap tm_out, const PairArgs args) {
    using L = PairSmem<STAGES>;
    using T = PairTmem<MODE>;
    constexpr uint32_t IDESC_F4 = idesc_nvf4_m(kPairTileM, kTileN);
    constexpr uint32_t IDESC_BF16 = idesc_bf16_m(kPairTileM, kTileN);
    constexpr uint32_t IDESC_BF16_HALF = idesc_bf16_m(kPairTileM, kTileN / 2);
    constexpr uint16_t kBoth = 0x3;
    constexpr uint32_t kAll = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);   // the leader's is used
    uint64_t* empty = full + STAGES;
    uint64_t* sf_full = empty + STAGES;            // this CTA's scale atoms are in shared memory
    uint64_t* sf_empty = sf_full + kPairSfStages;  // its staging warps have read them
    uint64_t* sf_ready = sf_empty + kPairSfStages; // the leader's: both CTAs staged a slot
    uint64_t* slot_free = sf_ready + L::MAX_SLOTS; // the MMAs that read a slot have completed
    uint64_t* tmem_full = slot_free + L::MAX_SLOTS;
    uint64_t* acc_empty = tmem_full + 1;                                // the leader's is used
    uint64_t* lacc_full = acc_empty + 1;           // raw: the second LoRA half is complete
    uint64_t* lacc_empty = lacc_full + 1;          // raw, the leader's: a LoRA half has been read
    uint64_t* drain = lacc_empty + 1;
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
        if (args.vec_out) prefetch_tensor_map(&tm_out);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);          // the leader's expect_tx; bytes from both CTAs
            mbar_init(&empty[s], 1);         // the leader's multicast commit
        }
        for (int s = 0; s < kPairSfStages; ++s) {
            mbar_init(&sf_full[s], 1);       // this CTA's scale producer; its own bulk copies
            mbar_init(&sf_empty[s], 4);      // this CTA's four staging warps
        }
        for (int k = 0; k < L::MAX_SLOTS; ++k) {
            mbar_init(&sf_ready[k], 2 * 4);  // the four staging warps of each CTA
            mbar_init(&slot_free[k], 1);     // the leader's multicast commit
        }
        mbar_init(tmem_full, 1);
        mbar_init(acc_empty, 2 * 32 * kEpiWarps);   // every epilogue thread of both CTAs
        mbar_init(lacc_full, 1);
        mbar_init(lacc_empty, 2 * 32 * (kEpiWarps / 2));   // one half's epilogue threads, both CTAs
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

    const int wg = warp >> 2;
    if (wg == 0) {
        reg_dealloc<kPairRegsCtl>();
        if (warp == 0 && lane == 0) {
            // ------------------------------- TMA producer (both CTAs) -------------------------------
            grid_dependency_wait();
            float sv = 0.0f;
            if constexpr (MODE != Mode::Off) sv = *args.scale;
            if (MODE != Mode::Off) {
                prefetch_tensor_map(&tm_d);
                prefetch_tensor_map(&tm_lb);
            }
            const bool lora_on = (MODE != Mode::Off) && sv != 0.0f;
            const bool bias_smem = args.bias != nullptr && args.vec_out;
            int stage = 0, tl = 0;
            uint32_t phase = 0, bias_issued = 0, bias_par = 0;
            bool ok = true;
            bool pend = false;                 // raw: the previous tile's LoRA half 1 is still due
            int prev_m = 0, prev_n = 0;
            // one ring item: wait for the stage, arm the leader's barrier, issue this CTA's loads
            auto next_stage = [&](uint32_t tx, uint32_t& lead_full, uint8_t*& sa, uint8_t*& sb) -> bool {
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) return false;
                lead_full = map_to_rank(smem_u32(&full[stage]), 0);
                sa = smem + L::A_OFF + stage * L::A_BYTES;
                sb = smem + L::B_OFF + stage * L::B_BYTES;
                if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * tx);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
                return true;
            };
            auto emit_base = [&](int it, int row_a, int row_b) -> bool {
                uint32_t lf; uint8_t *sa, *sb;
                if (!next_stage(L::STAGE_TX, lf, sa, sb)) return false;
                tma_load_2d_pair(sa, &tm_a, lf, it * 128, row_a);
                tma_load_2d_pair(sb, &tm_b, lf, it * 128, row_b);
                return true;
            };
            auto emit_lora = [&](int c, int row_a, int row_b) -> bool {   // prepared: d + lora_b rows
                uint32_t lf; uint8_t *sa, *sb;
                if (!next_stage(L::LORA_TX, lf, sa, sb)) return false;
                tma_load_2d_pair(sa, &tm_d, lf, c * 64, row_a);
                tma_load_2d_pair(sb, &tm_lb, lf, c * 64, row_b);
                return true;
            };
            // raw: d rows + this CTA's 64 lora_b rows of N-half h (64-row boxes)
            auto emit_half = [&](int c, int h, int m_pair, int n_blk) -> bool {
                uint32_t lf; uint8_t *sa, *sb;
                if (!next_stage(L::LORA_HALF_TX, lf, sa, sb)) return false;
                tma_load_2d_pair(sa, &tm_d, lf, c * 64, m_pair * kPairTileM + (int)rank * 128);
                tma_load_2d_pair(sb, &tm_lb, lf, c * 64, n_blk * kTileN + h * 128 + (int)rank * 64);
                return true;
            };
            for (int tile = pair; ok && tile < args.num_tiles; tile += npairs, ++tl) {
                const int m_pair = tile % args.m_pairs;
                const int n_blk = tile / args.m_pairs;
                const int row_a = m_pair * kPairTileM + (int)rank * 128;      // this CTA's A rows
                const int row_b = n_blk * kTileN + (int)rank * 128;           // this CTA's B half
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
                // ring items: base stages; raw: the previous tile's LoRA half 1 before base stage
                // kRawHalf1At (or after the base stages), this tile's half 0 after them; prepared:
                // the LoRA chunks after the base stages
                // (two segments around the half-1 point: no check for it in the per-stage loop)
                const int h1_at = min(kRawHalf1At, args.k_stages);
                int it = 0;
                for (int seg = 0; ok && seg < 2; ++seg) {
                    const int it_end = seg == 0 ? h1_at : args.k_stages;
                    for (; ok && it < it_end; ++it) ok = emit_base(it, row_a, row_b);
                    if (ok && seg == 0 && MODE == Mode::Raw && pend) {
                        for (int c = 0; ok && c < lora_chunks_if_on; ++c) ok = emit_half(c, 1, prev_m, prev_n);
                        pend = false;
                    }
                }
                if (ok && lora_on) {
                    if (MODE == Mode::Raw) {
                        for (int c = 0; ok && c < lora_chunks_if_on; ++c) ok = emit_half(c, 0, m_pair, n_blk);
                        pend = true;
                        prev_m = m_pair;
                        prev_n = n_blk;
                    } else {
                        for (int c = 0; ok && c < lora_chunks_if_on; ++c) ok = emit_lora(c, row_a, row_b);
                    }
                }
            }
            if (ok && MODE == Mode::Raw && pend)
                for (int c = 0; ok && c < lora_chunks_if_on; ++c) ok = emit_half(c, 1, prev_m, prev_n);
            if (!ok || *abort_flag) {
                // Let this CTA's own-barrier copies land before it can exit (the pair's code-tile
                // loads complete on the leader's barriers; both CTAs meet at the final cluster
                // barrier).
                for (int k = 0; k < 2; ++k)
                    if ((bias_issued >> k) & 1u) mbar_wait(&bias_full[k], (bias_par >> k) & 1u, nullptr);
            }
        } else if (warp == 2 && lane == 0) {
            // ------------------------- scale-atom producer (both CTAs) -------------------------
            // Per base K stage: this CTA's 4 A atoms (its 128-row block) and the 4 atoms of each of
            // the tile's two 128-row B blocks, 512 bytes each, into the scale ring.  A block past the
            // end of the scale buffer (rows past M or N only) is not copied: the TMEM columns it
            // would fill scale only rows whose codes are zero-filled and whose outputs are clipped.
            grid_dependency_wait();
            int sst = 0;
            uint32_t sphase = 0, issued = 0, issued_par = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < args.num_tiles; tile += npairs) {
                const int m_pair = tile % args.m_pairs;
                const int n_blk = tile / args.m_pairs;
                const int blk_a = m_pair * 2 + (int)rank;
                const bool has_a = blk_a < args.sf_row_blocks_a;
                const int rb0 = n_blk * 2;
                const int nsfb = (rb0 + 1 < args.sf_row_blocks_b) ? 2 : 1;
                for (int it = 0; it < args.k_stages; ++it) {
                    if (!mbar_wait(&sf_empty[sst], sphase ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&sf_full[sst], (has_a ? 2048u : 0u) + (uint32_t)nsfb * 2048u);
                    if (has_a)
                        bulk_load(smem + L::SFA_OFF + sst * L::SFA_BYTES,
                                  args.a_sf + ((size_t)blk_a * args.sf_atoms_k + it * 4) * 512, 2048, &sf_full[sst]);
                    uint8_t* sfb = smem + L::SFB_OFF + sst * L::SFB_BYTES;
                    for (int j = 0; j < nsfb; ++j)
                        bulk_load(sfb + j * 2048, args.b_sf + ((size_t)(rb0 + j) * args.sf_atoms_k + it * 4) * 512,
                                  2048, &sf_full[sst]);
                    issued |= 1u << sst;
                    issued_par = (issued_par & ~(1u << sst)) | (sphase << sst);
                    if (++sst == kPairSfStages) { sst = 0; sphase ^= 1; }
                }
            }
            if (!ok || *abort_flag) {
                // Let the copies already issued land before the CTA can exit.
                for (int k = 0; k < kPairSfStages; ++k)
                    if ((issued >> k) & 1u) mbar_wait(&sf_full[k], (issued_par >> k) & 1u, nullptr);
            }
        } else if (warp == 1 && lane == 0 && rank == 0) {
            // ------------------------------- MMA issuer (the leader) -------------------------------
            grid_dependency_wait();
            float sv = 0.0f;
            if constexpr (MODE != Mode::Off) sv = *args.scale;
            const bool lora_on = (MODE != Mode::Off) && sv != 0.0f;
            int stage = 0, slot = 0;
            uint32_t phase = 0, slot_use = 0, lacc_waits = 0;
            bool ok = true;
            // Raw path: one LoRA half of a tile, one ring item per 64-rank chunk (d rows and this
            // CTA's 64 lora_b rows of the half), into the LoRA accumulator (M = 256, N = 128).
            auto lora_half = [&]() -> bool {
                for (int c = 0; c < lora_chunks_if_on; ++c) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) return false;
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                    const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                    const int rem = args.r - c * 64;
                    const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                    for (int j = 0; j < ksteps; ++j)
                        tc_mma_bf16_pair(tmem + T::LACC, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                         IDESC_BF16_HALF, (c > 0 || j > 0) ? 1u : 0u);
                    tc_commit_pair_multicast(&empty[stage], kBoth);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                return true;
            };
            // Raw path: the previous tile's half 1, once the epilogue warps of half 0 (both CTAs)
            // have read the LoRA accumulator; issued kRawHalf1At stages into the next tile so that
            // the tensor pipe does not idle meanwhile.
            bool pend = false;
            auto finish_pending = [&]() -> bool {
                if (!mbar_wait_cluster(lacc_empty, (lacc_waits++ & 1) ^ 1, abort_flag)) return false;
                tc_fence_after();
                if (!lora_half()) return false;
                tc_commit_pair_multicast(lacc_full, kBoth);
                pend = false;
                return true;
            };
            const int h1_at = min(kRawHalf1At, args.k_stages);
            int i = 0;
            for (int tile = pair; ok && tile < args.num_tiles; tile += npairs, ++i) {
                // both CTAs' epilogues have read the previous tile's accumulator
                if (!mbar_wait_cluster(acc_empty, (i & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                // the base stages, in two segments around the half-1 point so that the issue loop
                // itself carries no check for it (one there cost about 4 % in the raw kernel)
                int it = 0;
                for (int seg = 0; ok && seg < 2; ++seg) {
                    const int it_end = seg == 0 ? h1_at : args.k_stages;
                    for (; it < it_end; ++it) {
                        // both CTAs staged this slot's scales, and both CTAs' code tiles landed
                        if (!mbar_wait_cluster(&sf_ready[slot], slot_use & 1u, abort_flag)) { ok = false; break; }
                        if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                        const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                        const uint32_t sfa_t = tmem + T::SF0 + slot * T::SLOT_COLS;
                        const uint32_t sfb_t = sfa_t + T::SFA_COLS;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc_mma_nvf4_pair(tmem + T::ACC, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                             IDESC_F4, sfa_t + 4 * j, sfb_t + 8 * j, (it > 0 || j > 0) ? 1u : 0u);
                        tc_commit_pair_multicast(&empty[stage], kBoth);
                        tc_commit_pair_multicast(&slot_free[slot], kBoth);
                        if (++slot == T::NSF) { slot = 0; ++slot_use; }
                        if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    }
                    if (ok && seg == 0 && MODE == Mode::Raw && pend && !finish_pending()) ok = false;
                }
                if (!ok) break;
                if (lora_on && MODE == Mode::Prepared) {
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
                    tc_commit_pair_multicast(tmem_full, kBoth);   // both CTAs' accumulators are complete
                } else if (lora_on && MODE == Mode::Raw) {
                    // raw LoRA half 0 in its own accumulator, once the previous tile's half 1 has
                    // been read
                    if (!mbar_wait_cluster(lacc_empty, (lacc_waits++ & 1) ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (!lora_half()) { ok = false; break; }
                    tc_commit_pair_multicast(tmem_full, kBoth);   // base accumulator + LoRA half 0
                    pend = true;
                } else {
                    tc_commit_pair_multicast(tmem_full, kBoth);   // both CTAs' accumulators are complete
                }
            }
            if (ok && MODE == Mode::Raw && pend && !finish_pending()) ok = false;
            if (!ok || *abort_flag) {
                // Wait for the MMAs already issued before TMEM is released.
                tc_commit_pair_multicast(drain, 0x1);
                mbar_wait(drain, 0, nullptr);
            }
        }
        __syncwarp();
    } else if (wg == 1) {
        reg_dealloc<kPairRegsStage>();
        // ------------------------------- scale staging (both CTAs) -------------------------------
        // Per base K stage: this warp's TMEM lane quarter gets the 12 atoms' row `lane` (16 bytes
        // each) as 4 columns per atom; the A atoms first (K steps 0..3), then per K step the two
        // 128-row blocks of B.  Every lane quarter holds the whole atom, as a warpx4 copy leaves it.
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        grid_dependency_wait();
        const uint32_t lead_sf_ready = map_to_rank(smem_u32(sf_ready), 0);
        int sst = 0;
        uint32_t sphase = 0, g = 0;
        bool ok = true;
        for (int tile = pair; ok && tile < args.num_tiles; tile += npairs) {
            for (int it = 0; it < args.k_stages; ++it) {
                const uint32_t slot = g % T::NSF, use = g / T::NSF;
                if (!__all_sync(kAll, mbar_wait(&sf_full[sst], sphase, abort_flag))) { ok = false; break; }
                const uint8_t* srca = smem + L::SFA_OFF + sst * L::SFA_BYTES + lane * 16;
                const uint8_t* srcb = smem + L::SFB_OFF + sst * L::SFB_BYTES + lane * 16;
                uint32_t va[16], vb[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 w = *reinterpret_cast<const uint4*>(srca + j * 512);
                    va[4 * j] = w.x; va[4 * j + 1] = w.y; va[4 * j + 2] = w.z; va[4 * j + 3] = w.w;
                    const uint4 w0 = *reinterpret_cast<const uint4*>(srcb + j * 512);
                    const uint4 w1 = *reinterpret_cast<const uint4*>(srcb + 2048 + j * 512);
                    vb[8 * j] = w0.x; vb[8 * j + 1] = w0.y; vb[8 * j + 2] = w0.z; vb[8 * j + 3] = w0.w;
                    vb[8 * j + 4] = w1.x; vb[8 * j + 5] = w1.y; vb[8 * j + 6] = w1.z; vb[8 * j + 7] = w1.w;
                }
                // the slot's previous MMAs have completed (its loads overlap this wait)
                if (use > 0 && !__all_sync(kAll, mbar_wait(&slot_free[slot], (use - 1) & 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t col = tmem + lane_off + T::SF0 + slot * T::SLOT_COLS;
                tmem_store_16(col, va);
                tmem_store_32(col + T::SFA_COLS, vb);
                // the stores have read their registers, so the loads are done: the ring slot is free
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_empty[sst]);
                tmem_store_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote_relaxed(lead_sf_ready + slot * 8);
                ++g;
                if (++sst == kPairSfStages) { sst = 0; sphase ^= 1; }
            }
        }
    } else {
        reg_alloc<kPairRegsEpi>();
        // ------------------------------- epilogue (both CTAs) -------------------------------
        const int ew = warp - 8;                       // epilogue warp 0..7
        const int q = warp & 3;                        // TMEM lane quarter of this warp
        const int h = ew >> 2;                         // which 128 of the 256 columns
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        grid_dependency_wait();
        float lora_s = 0.0f;
        if constexpr (MODE == Mode::Raw) lora_s = *args.scale;
        const bool raw_lora = (MODE == Mode::Raw) && lora_s != 0.0f;
        const float alpha = *args.alpha;
        const uint32_t lead_acc_empty = map_to_rank(smem_u32(acc_empty), 0);
        const uint32_t lead_lacc_empty = map_to_rank(smem_u32(lacc_empty), 0);
        int i = 0, out_box = 0;
        for (int tile = pair; tile < args.num_tiles; tile += npairs, ++i) {
            const int m_pair = tile % args.m_pairs;
            const int n_blk = tile / args.m_pairs;
            if (!__all_sync(kAll, mbar_wait(tmem_full, i & 1, abort_flag))) break;
            tc_fence_after();
            uint32_t raw[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_load_32(tmem + lane_off + T::ACC + h * 128 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(raw + c * 32));
            tmem_load_wait();
            tc_fence_before();
            // the leader may start the next tile's MMAs once both CTAs hold their accumulators
            // (tcgen05.wait::ld has returned, so the arrival carries no data: relaxed suffices)
            if (rank == 0) mbar_arrive(acc_empty);
            else mbar_arrive_remote_relaxed(lead_acc_empty);
            float v[128];
#pragma unroll
            for (int k = 0; k < 128; ++k) v[k] = __fmul_rn(alpha, __uint_as_float(raw[k]));
            if (MODE == Mode::Raw && raw_lora) {
                // half 0 of the LoRA accumulator is complete with the base one (tmem_full); half 1
                // once lacc_full says so, after the h = 0 warps of both CTAs have released half 0
                if (h == 1 && !__all_sync(kAll, mbar_wait(lacc_full, i & 1, abort_flag))) break;
                tc_fence_after();
                // 16 columns at a time: with the 128 held values this keeps the epilogue within
                // its registers (32-column reads spilled)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t lv[16];
                    tmem_load_16(tmem + lane_off + T::LACC + c * 16, lv);
                    tmem_load_wait();
#pragma unroll
                    for (int k = 0; k < 16; ++k) v[c * 16 + k] = __fmaf_rn(lora_s, __uint_as_float(lv[k]), v[c * 16 + k]);
                }
                tc_fence_before();
                if (rank == 0) mbar_arrive(lacc_empty);
                else mbar_arrive_remote_relaxed(lead_lacc_empty);
            }
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
                uint8_t* box0 = smem + L::OUT_OFF + ew * kPairOutBoxes * L::OUT_BOX_BYTES;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint8_t* box = box0 + out_box * L::OUT_BOX_BYTES;
                    if (++out_box == kPairOutBoxes) out_box = 0;
                    if (lane == 0) bulk_wait_group_read<kPairOutBoxes - 1>();   // its previous store has read it
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
