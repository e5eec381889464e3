// Persistent warp-specialised NVFP4 x NVFP4 GEMM with a fused BF16 LoRA term (sm_100a).
//
// Computes flashinfer.gemm.mm_nvfp4_lora's opening formula
//     out = bf16_rne(alpha * (dequant(a) @ dequant(b)^T) + lora_scale * (d @ lora_b^T) [+ bias])
// one 128 x 256 output tile at a time, tiles strided over a persistent grid.  Four warpgroups:
//   warpgroup 0  warp 0: TMA producer of the A/B code tiles (2-D TMA, 128-byte swizzle) per
//                256-wide K stage and, after a tile's base stages, of the d / lora_b tiles of
//                the LoRA term (64 ranks per stage).  Warp 1: allocates TMEM; one thread issues
//                the block-scaled MMAs (kind::mxf4nvf4, 16-element UE4M3 scale vectors, M=128,
//                N=256) into a 256-column fp32 accumulator, then the bf16 MMAs (kind::f16,
//                K = r) of the LoRA term: on the prepared path into the accumulator after the
//                base product ("Prepared path" bullet); on the raw path into a separate 128-
//                column accumulator, one N-half at a time ("Raw path" bullet: alpha and
//                lora_scale stay independent).  Warp 2: bulk-copies each K stage's 512-byte
//                scale atoms into a ring of its own.
//   warpgroup 1  one warp per TMEM lane quarter: writes each stage's scale atoms from shared
//                memory into a TMEM scale slot with tcgen05.st (the layout a 32x128b.warpx4
//                copy of the atom gives), up to NSF stages ahead of the MMAs, so the MMA thread
//                issues nothing but MMAs.  A tcgen05.cp scale copy would share the tensor pipe
//                with the MMAs; a register store does not.
//   warpgroups 2-3  two warps per TMEM lane quarter: once a tile's accumulator is complete each
//                warp drains its 128 of the 256 columns with tcgen05.ld, releases the
//                accumulator (so the next tile's MMAs start), then v = alpha*acc
//                [; v = fma(s, lora_acc, v)] [; v += bias], one round-to-nearest-even to bf16 and
//                TMA stores.
// Registers are split by warpgroup (setmaxnreg).  N = 256 per MMA instruction halves the A-tile
// traffic per flop against N = 128.  Zero-adapter path (Parameters: lora_scale): every role reads
// the LoRA scalar; when it equals 0 no LoRA tile is loaded or multiplied and the epilogue is the
// adapter-off one, so the output is bitwise the adapter-off output.
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
    int vec_out;             // 1: rows of out (and bias) may be written / read 16 bytes at a time
    // grouped call (the GROUPED instantiation only): expert e owns rows [m_indptr[e],
    // m_indptr[e+1]) of a, d and out, rows [e*N, (e+1)*N) of b and lora_b, scale blocks
    // [e*sf_row_blocks_b, (e+1)*sf_row_blocks_b) of b_sf, alpha[e] and bias[e*N, (e+1)*N)
    const int* m_indptr;     // [num_experts + 1], device; multiples of 128, read on the device
    int num_experts;
};

constexpr int kMaxExperts = 511;         // grouped call: m_indptr lives in shared memory
constexpr int kErrBadIndptr = 2;         // device error word: a grouped call's m_indptr broke its rules

// Largest e in [0, E) with ind[e] <= row, for non-decreasing ind with ind[0] <= row < ind[E]: the
// expert whose rows hold `row` (empty experts, ind[e] == ind[e + 1], are skipped).
__device__ __forceinline__ int expert_of_row(const int* ind, int E, int row) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ind[mid] <= row) lo = mid; else hi = mid;
    }
    return lo;
}

constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kEpiWarps = 8;
constexpr int kOutBoxCols = 32;          // TMA store box of the epilogue: 32 columns x 32 rows
constexpr int kOutBoxRows = 32;
// Output staging: one 32 x 32 box per epilogue warp, rewritten once its previous store has read it
// (the epilogue has slack).  Against three boxes: the 8-expert grouped layer 37.5 us per call
// against 38.8, the M = 64 and 96 calls within 1 %.
constexpr int kOutBoxes = 1;
constexpr int kSfStages = 4;             // scale-atom ring (own barriers, recycled by the staging warps)
constexpr int kGemmThreads = 512;        // 4 warpgroups: producers/MMA, staging, 2 x epilogue
// Registers per thread after the split.  The block is launched with 512 x 128; the split must not
// exceed that pool (setmaxnreg.inc waits for registers that the other warpgroups give back).
constexpr int kGemmRegsLaunch = 128;
constexpr int kGemmRegsCtl = 80;         // warpgroup 0: producers, MMA issuer, one idle warp
constexpr int kGemmRegsStage = 72;       // warpgroup 1: scale staging
constexpr int kGemmRegsEpi = 176;        // warpgroups 2 and 3: epilogue
static_assert(128 * (kGemmRegsCtl + kGemmRegsStage) + 256 * kGemmRegsEpi <= kGemmThreads * kGemmRegsLaunch,
              "register split exceeds the launch's register pool");

// Shared-memory plan of one CTA.  Each stage holds one A tile (128 rows x 128 bytes) and one B
// tile (256 rows x 128 bytes); a LoRA stage reuses them for a 128 x 64 bf16 d tile and a 256 x 64
// bf16 lora_b tile (also 128 bytes per row).  The scale atoms of a stage sit in a ring of their own.
template <int STAGES>
struct GemmSmem {
    static constexpr int A_BYTES = kTileM * 128;
    static constexpr int B_BYTES = kTileN * 128;
    static constexpr int SFA_BYTES = 4 * 512;
    static constexpr int SFB_BYTES = (kTileN / 128) * 4 * 512;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int SFA_OFF = B_OFF + STAGES * B_BYTES;
    static constexpr int SFB_OFF = SFA_OFF + kSfStages * SFA_BYTES;
    // the tile's 256 bias values (bf16), double-buffered across tiles
    static constexpr int BIAS_BYTES = kTileN * 2;
    static constexpr int BIAS_OFF = SFB_OFF + kSfStages * SFB_BYTES;
    // per epilogue warp, kOutBoxes 32 x 32 bf16 output boxes for TMA stores, used round-robin
    static constexpr int OUT_BOX_BYTES = kOutBoxCols * kOutBoxRows * 2;
    static constexpr int OUT_OFF = BIAS_OFF + 2 * BIAS_BYTES;
    static constexpr int BAR_OFF = OUT_OFF + kEpiWarps * kOutBoxes * OUT_BOX_BYTES;
    static constexpr int MAX_SLOTS = 8;                  // TMEM scale slots (at most)
    // grouped call: m_indptr copied from global memory, then [rows / 128 in use, valid]
    static constexpr int IND_OFF = BAR_OFF;
    static constexpr int IND_BYTES = (kMaxExperts + 1) * 4 + 16;
    // full[S], empty[S], sf_full[SF], sf_empty[SF], sf_ready[8], slot_free[8], tmem_full,
    // acc_empty, lacc_full, lacc_empty, drain, bias_full[2], bias_empty[2], groups_ready
    static constexpr int NUM_BARS = 2 * STAGES + 2 * kSfStages + 2 * MAX_SLOTS + 10;
    static constexpr int MISC_OFF = BAR_OFF + IND_BYTES + NUM_BARS * 8;
    static constexpr int TOTAL = MISC_OFF + 16;
    static constexpr int DYN_BYTES = TOTAL + 1024;    // slack to align the base to 1024 bytes
    static_assert(DYN_BYTES <= 232448, "shared-memory plan exceeds 227 KB");
};

// TMEM plan (columns of 32-bit cells, 128 lanes): the 256-column accumulator, NSF scale slots
// used round-robin by the base K stages, and the raw path's 128-column LoRA accumulator.  A slot
// is rewritten only after the commit that follows the MMAs of its previous stage (slot_free).
template <Mode MODE>
struct TmemPlan {
    static constexpr int ACC = 0;
    static constexpr int SF0 = kTileN;
    static constexpr int SFA_COLS = 4 * 4;                // 4 MMAs (K = 64 each) x 4 columns
    static constexpr int SFB_COLS = 4 * (kTileN / 32);    // 4 MMAs x 8 columns
    static constexpr int SLOT_COLS = SFA_COLS + SFB_COLS;
    // more slots let the staging run further ahead of the MMAs still reading older slots
    static constexpr int NSF = (MODE == Mode::Raw) ? 2 : 5;
    static constexpr int LACC = SF0 + NSF * SLOT_COLS;    // raw path: 352
    static constexpr int USED = (MODE == Mode::Raw) ? LACC + 128 : LACC;
    static constexpr int ALLOC = 512;
    static_assert(USED <= ALLOC, "TMEM plan exceeds 512 columns");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int STAGES, Mode MODE, bool GROUPED = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_lb,
                  const __grid_constant__ CUtensorMap tm_out, const GemmArgs args) {
    using L = GemmSmem<STAGES>;
    using T = TmemPlan<MODE>;
    static_assert(T::NSF <= L::MAX_SLOTS, "scale slots exceed the barrier plan");
    constexpr uint32_t IDESC_F4 = idesc_nvf4(kTileN);
    constexpr uint32_t IDESC_BF16_FULL = idesc_bf16(kTileN);
    constexpr uint32_t IDESC_BF16_HALF = idesc_bf16(kTileN / 2);
    constexpr uint32_t kAll = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF + L::IND_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_full = empty + STAGES;           // a stage's scale atoms are in shared memory
    uint64_t* sf_empty = sf_full + kSfStages;     // ... and the staging warps have read them
    uint64_t* sf_ready = sf_empty + kSfStages;    // a slot holds its stage's scales in TMEM
    uint64_t* slot_free = sf_ready + L::MAX_SLOTS;  // the MMAs that read a slot have completed
    uint64_t* tmem_full = slot_free + L::MAX_SLOTS;
    uint64_t* acc_empty = tmem_full + 1;
    uint64_t* lacc_full = acc_empty + 1;
    uint64_t* lacc_empty = lacc_full + 1;
    uint64_t* drain = lacc_empty + 1;
    uint64_t* bias_full = drain + 1;              // [2]: a tile's bias values are in shared memory
    uint64_t* bias_empty = bias_full + 2;         // [2]: ... and every epilogue thread has read them
    uint64_t* groups_ready = bias_empty + 2;      // grouped call: m_indptr is in shared memory
    int* ind = reinterpret_cast<int*>(smem + L::IND_OFF);   // grouped: m_indptr, then [m_tiles, valid]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int lora_chunks_if_on = (args.r + 63) / 64;

    if (threadIdx.x == 0) {
        prefetch_tensor_map(&tm_a);
        prefetch_tensor_map(&tm_b);
        if (args.vec_out) prefetch_tensor_map(&tm_out);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kSfStages; ++s) {
            mbar_init(&sf_full[s], 1);
            mbar_init(&sf_empty[s], 4);                // the 4 staging warps
        }
        for (int k = 0; k < T::NSF; ++k) {
            mbar_init(&sf_ready[k], 4);                // the 4 staging warps
            mbar_init(&slot_free[k], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(acc_empty, 32 * kEpiWarps);
        mbar_init(lacc_full, 1);
        mbar_init(lacc_empty, 128);
        mbar_init(drain, 1);
        for (int k = 0; k < 2; ++k) {
            mbar_init(&bias_full[k], 1);
            mbar_init(&bias_empty[k], 32 * kEpiWarps);
        }
        mbar_init(groups_ready, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, T::ALLOC);
        tmem_relinquish();
    }
    const int E = GROUPED ? args.num_experts : 1;
    // The tile grid: (m blocks of 128 rows) x (n blocks of 256 columns), m fastest.  A grouped call
    // takes its rows, [0, m_indptr[E]), from the table warp 3 puts in shared memory (no tiles at all
    // when m_indptr breaks its rules); every role reads the same values.
    auto tile_grid = [&](int& m_tiles, int& num_tiles) -> bool {
        if constexpr (!GROUPED) {
            m_tiles = args.m_tiles;
            num_tiles = args.num_tiles;
            return true;
        } else {
            m_tiles = 0;
            num_tiles = 0;
            if (!mbar_wait(groups_ready, 0, abort_flag)) return false;
            m_tiles = ind[kMaxExperts + 1];
            num_tiles = m_tiles * args.n_tiles;
            return true;
        }
    };
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Programmatic dependent launch: the next kernel on the stream may start its own prologue
    // now; every access to memory another kernel may write comes after grid_dependency_wait().
    grid_launch_dependents();

    const int wg = warp >> 2;
    if (wg == 0) {
        reg_dealloc<kGemmRegsCtl>();
        if (warp == 0 && lane == 0) {
            // ------------------------------- TMA producer -------------------------------
            if (!GROUPED && blockIdx.x < args.num_tiles) {
                // warm L2 with the first stages of this CTA's first tile (a prefetch changes no
                // data, so it may precede the dependency wait)
                const int m_blk = blockIdx.x % args.m_tiles, n_blk = blockIdx.x / args.m_tiles;
                for (int it = 0; it < STAGES && it < args.k_stages; ++it) {
                    tma_prefetch_l2_2d(&tm_a, it * 128, m_blk * kTileM);
                    tma_prefetch_l2_2d(&tm_b, it * 128, n_blk * kTileN);
                }
            }
            grid_dependency_wait();
            float sv = 0.0f;
            if constexpr (MODE != Mode::Off) sv = *args.scale;   // consumed after the base stages
            if (MODE != Mode::Off) {
                prefetch_tensor_map(&tm_d);
                prefetch_tensor_map(&tm_lb);
            }
            int stage = 0;
            uint32_t phase = 0, filled = 0, filled_parity = 0;
            int m_tiles, num_tiles;
            bool ok = tile_grid(m_tiles, num_tiles);
            const bool bias_smem = args.bias != nullptr && args.vec_out;
            int tl = 0;                                // local tile counter
            uint32_t bias_issued = 0, bias_par = 0;    // per buffer: issued, parity of its last phase
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++tl) {
                const int m_blk = tile % m_tiles;
                const int n_blk = tile / m_tiles;
                const int e = GROUPED ? expert_of_row(ind, E, m_blk * kTileM) : 0;
                const int b_row = e * args.N + n_blk * kTileN;     // this tile's rows of b / lora_b
                const int items = args.k_stages + (sv != 0.0f ? lora_chunks_if_on : 0);
                if (bias_smem) {
                    // the tile's bias slice, once the epilogue of two tiles ago has read the buffer
                    const int bb = tl & 1;
                    if (!mbar_wait(&bias_empty[bb], ((tl >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    const int n0 = n_blk * kTileN;
                    const uint32_t bytes = (uint32_t)min(kTileN, args.N - n0) * 2u;   // N % 8 == 0
                    mbar_arrive_expect_tx(&bias_full[bb], bytes);
                    bulk_load(smem + L::BIAS_OFF + bb * L::BIAS_BYTES, args.bias + (size_t)e * args.N + n0, bytes,
                              &bias_full[bb]);
                    bias_issued |= 1u << bb;
                    bias_par = (bias_par & ~(1u << bb)) | ((((uint32_t)tl >> 1) & 1u) << bb);
                }
                for (int it = 0; it < items; ++it) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* sa = smem + L::A_OFF + stage * L::A_BYTES;
                    uint8_t* sb = smem + L::B_OFF + stage * L::B_BYTES;
                    mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
                    if (it >= args.k_stages) {
                        const int c = it - args.k_stages;
                        tma_load_2d(sa, &tm_d, &full[stage], c * 64, m_blk * kTileM);
                        tma_load_2d(sb, &tm_lb, &full[stage], c * 64, b_row);
                    } else {
                        tma_load_2d(sa, &tm_a, &full[stage], it * 128, m_blk * kTileM);
                        tma_load_2d(sb, &tm_b, &full[stage], it * 128, b_row);
                    }
                    filled |= 1u << stage;
                    filled_parity = (filled_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok || *abort_flag) {
                // Let every copy already issued land before the CTA can exit.
                for (int k = 0; k < 2; ++k)
                    if ((bias_issued >> k) & 1u) mbar_wait(&bias_full[k], (bias_par >> k) & 1u, nullptr);
                for (int s = 0; s < STAGES; ++s)
                    if ((filled >> s) & 1u) mbar_wait(&full[s], (filled_parity >> s) & 1u, nullptr);
            }
        } else if (warp == 2 && lane == 0) {
            // ------------------------------ scale-atom producer ------------------------------
            // Per base K stage: the 4 A atoms of the tile's 128-row block and the 4 atoms of each
            // of its two 128-row B blocks, 512 bytes each.  A B block past the end of b_sf (rows
            // past N only) is not copied: the TMEM columns it would fill scale only rows whose
            // codes are zero-filled and whose outputs are clipped.
            grid_dependency_wait();
            int sst = 0;
            uint32_t sphase = 0, issued = 0, issued_par = 0;
            int m_tiles, num_tiles;
            bool ok = tile_grid(m_tiles, num_tiles);
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const int m_blk = tile % m_tiles;
                const int n_blk = tile / m_tiles;
                const int e = GROUPED ? expert_of_row(ind, E, m_blk * kTileM) : 0;
                const int rbl = n_blk * (kTileN / 128);     // the tile's first 128-row block of B
                const int nsfb = (rbl + 1 < args.sf_row_blocks_b) ? 2 : 1;
                const int rb0 = e * args.sf_row_blocks_b + rbl;
                for (int it = 0; it < args.k_stages; ++it) {
                    if (!mbar_wait(&sf_empty[sst], sphase ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&sf_full[sst], 2048u + (uint32_t)nsfb * 2048u);
                    bulk_load(smem + L::SFA_OFF + sst * L::SFA_BYTES,
                              args.a_sf + ((size_t)m_blk * args.sf_atoms_k + it * 4) * 512, 2048, &sf_full[sst]);
                    uint8_t* sfb = smem + L::SFB_OFF + sst * L::SFB_BYTES;
                    for (int j = 0; j < nsfb; ++j)
                        bulk_load(sfb + j * 2048, args.b_sf + ((size_t)(rb0 + j) * args.sf_atoms_k + it * 4) * 512,
                                  2048, &sf_full[sst]);
                    issued |= 1u << sst;
                    issued_par = (issued_par & ~(1u << sst)) | (sphase << sst);
                    if (++sst == kSfStages) { sst = 0; sphase ^= 1; }
                }
            }
            if (!ok || *abort_flag) {
                // Let the copies already issued land before the CTA can exit.
                for (int k = 0; k < kSfStages; ++k)
                    if ((issued >> k) & 1u) mbar_wait(&sf_full[k], (issued_par >> k) & 1u, nullptr);
            }
        } else if (warp == 1 && lane == 0) {
            // ------------------------------- MMA issuer ---------------------------------
            grid_dependency_wait();
            float sv = 0.0f;
            if constexpr (MODE != Mode::Off) sv = *args.scale;
            int stage = 0, slot = 0;
            uint32_t phase = 0, slot_use = 0, lacc_waits = 0;
            int m_tiles, num_tiles;
            bool ok = tile_grid(m_tiles, num_tiles);
            int i = 0;   // local tile counter
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++i) {
                if (!mbar_wait(acc_empty, (i & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                // base product: k_stages x 4 MMAs of 128 x 256 x 64
                for (int it = 0; ok && it < args.k_stages; ++it) {
                    if (!mbar_wait(&sf_ready[slot], slot_use & 1u, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                    const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                    const uint32_t sfa_t = tmem + T::SF0 + slot * T::SLOT_COLS;
                    const uint32_t sfb_t = sfa_t + T::SFA_COLS;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc_mma_nvf4(tmem + T::ACC, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                    IDESC_F4, sfa_t + 4 * j, sfb_t + 8 * j, (it > 0 || j > 0) ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    tc_commit(&slot_free[slot]);
                    if (++slot == T::NSF) { slot = 0; ++slot_use; }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                const bool lora_on = (MODE != Mode::Off) && sv != 0.0f;
                if (lora_on && MODE == Mode::Prepared) {
                    // folded LoRA term into the same accumulator, after the base product
                    for (int c = 0; ok && c < lora_chunks_if_on; ++c) {
                        if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + L::A_OFF + stage * L::A_BYTES);
                        const uint32_t b_addr = smem_u32(smem + L::B_OFF + stage * L::B_BYTES);
                        const int rem = args.r - c * 64;
                        const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                        for (int j = 0; j < ksteps; ++j)
                            tc_mma_bf16(tmem + T::ACC, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                        IDESC_BF16_FULL, 1u);
                        tc_commit(&empty[stage]);
                        if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    }
                    if (!ok) break;
                    tc_commit(tmem_full);
                } else if (lora_on && MODE == Mode::Raw) {
                    // raw LoRA term in its own 128-column accumulator, one N-half at a time; the
                    // chunks' shared-memory stages stay held until the second half is issued
                    int st0 = 0, st1 = 0;      // stages of LoRA chunks 0 and 1 (r <= 128)
                    for (int c = 0; ok && c < lora_chunks_if_on; ++c) {
                        if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                        if (c == 0) st0 = stage; else st1 = stage;
                        if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    }
                    if (ok && !mbar_wait(lacc_empty, (lacc_waits++ & 1) ^ 1, abort_flag)) ok = false;
                    if (!ok) break;
                    tc_fence_after();
                    for (int half = 0; half < 2; ++half) {
                        if (half == 1) {
                            tc_commit(tmem_full);      // base accumulator + LoRA half 0 are ready
                            if (!mbar_wait(lacc_empty, (lacc_waits++ & 1) ^ 1, abort_flag)) { ok = false; break; }
                            tc_fence_after();
                        }
                        for (int c = 0; c < lora_chunks_if_on; ++c) {
                            const int stc = (c == 0) ? st0 : st1;
                            const uint32_t a_addr = smem_u32(smem + L::A_OFF + stc * L::A_BYTES);
                            const uint32_t b_addr = smem_u32(smem + L::B_OFF + stc * L::B_BYTES) + half * (128 * 128);
                            const int rem = args.r - c * 64;
                            const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                            for (int j = 0; j < ksteps; ++j)
                                tc_mma_bf16(tmem + T::LACC, sdesc_sw128(a_addr + j * 32), sdesc_sw128(b_addr + j * 32),
                                            IDESC_BF16_HALF, (c > 0 || j > 0) ? 1u : 0u);
                        }
                    }
                    if (!ok) break;
                    tc_commit(lacc_full);
                    tc_commit(&empty[st0]);
                    if (lora_chunks_if_on > 1) tc_commit(&empty[st1]);
                } else {
                    tc_commit(tmem_full);
                }
            }
            if (!ok || *abort_flag) {
                // Wait for the MMAs already issued before TMEM is released.
                tc_commit(drain);
                mbar_wait(drain, 0, nullptr);
            }
        } else if (GROUPED && warp == 3) {
            // --------------------- grouped call: m_indptr into shared memory ---------------------
            // Its rules (the grouped reading of the 128x4 layout): m_indptr[0] == 0, non-decreasing,
            // every entry a multiple of 128 and at most M (the rows of a, d and out).  A table that
            // breaks them gives no tiles and raises the device error word.
            grid_dependency_wait();
            bool valid = true;
            for (int k = lane; k <= E; k += 32) {
                const int v = args.m_indptr[k];
                ind[k] = v;
                if (v < 0 || v % kTileM != 0 || v > args.M) valid = false;
                if (k == 0 && v != 0) valid = false;
                if (k > 0 && v < args.m_indptr[k - 1]) valid = false;
            }
            valid = __all_sync(kAll, valid);
            __syncwarp();
            if (lane == 0) {
                ind[kMaxExperts + 1] = valid ? ind[E] / kTileM : 0;
                if (!valid) atomicExch(&g_device_error, kErrBadIndptr);
                mbar_arrive(groups_ready);
            }
        }
        __syncwarp();
    } else if (wg == 1) {
        reg_dealloc<kGemmRegsStage>();
        // ------------------------------- scale staging -------------------------------
        // Per base K stage: this warp's TMEM lane quarter gets the 12 atoms' row `lane` (16 bytes
        // each) as 4 columns per atom; the A atoms first (K steps 0..3), then per K step the two
        // 128-row blocks of B.  Every lane quarter holds the whole atom, as a warpx4 copy leaves it.
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        grid_dependency_wait();
        int sst = 0;
        uint32_t sphase = 0, g = 0;
        int m_tiles, num_tiles;
        bool ok = __all_sync(kAll, tile_grid(m_tiles, num_tiles));
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            for (int it = 0; it < args.k_stages; ++it) {
                const uint32_t slot = g % T::NSF, use = g / T::NSF;
                if (!__all_sync(kAll, mbar_wait(&sf_full[sst], sphase, abort_flag))) { ok = false; break; }
                const uint8_t* srca = smem + L::SFA_OFF + sst * L::SFA_BYTES + lane * 16;
                const uint8_t* srcb = smem + L::SFB_OFF + sst * L::SFB_BYTES + lane * 16;
                uint32_t va[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 w = *reinterpret_cast<const uint4*>(srca + j * 512);
                    va[4 * j] = w.x; va[4 * j + 1] = w.y; va[4 * j + 2] = w.z; va[4 * j + 3] = w.w;
                }
                // the slot's previous MMAs have completed (the A loads overlap this wait; the B atoms
                // are read after it, which keeps the warp within its 72 registers)
                if (use > 0 && !__all_sync(kAll, mbar_wait(&slot_free[slot], (use - 1) & 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t col = tmem + lane_off + T::SF0 + slot * T::SLOT_COLS;
                tmem_store_16(col, va);
                uint32_t vb[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 w0 = *reinterpret_cast<const uint4*>(srcb + j * 512);
                    const uint4 w1 = *reinterpret_cast<const uint4*>(srcb + 2048 + j * 512);
                    vb[8 * j] = w0.x; vb[8 * j + 1] = w0.y; vb[8 * j + 2] = w0.z; vb[8 * j + 3] = w0.w;
                    vb[8 * j + 4] = w1.x; vb[8 * j + 5] = w1.y; vb[8 * j + 6] = w1.z; vb[8 * j + 7] = w1.w;
                }
                tmem_store_32(col + T::SFA_COLS, vb);
                // the stores have read their registers, so the loads are done: the ring slot is free
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_empty[sst]);
                tmem_store_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[slot]);
                ++g;
                if (++sst == kSfStages) { sst = 0; sphase ^= 1; }
            }
        }
    } else {
        reg_alloc<kGemmRegsEpi>();
        // ------------------------------- epilogue -------------------------------
        const int ew = warp - 8;                       // epilogue warp 0..7
        const int q = warp & 3;                        // TMEM lane quarter of this warp
        const int h = ew >> 2;                         // which 128 of the 256 columns
        const int rl = q * 32 + lane;                  // row within the tile
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        grid_dependency_wait();
        float lora_s = 0.0f;
        if constexpr (MODE != Mode::Off) lora_s = *args.scale;
        const bool lora_on = (MODE != Mode::Off) && lora_s != 0.0f;
        const float alpha0 = *args.alpha;
        int m_tiles, num_tiles;
        const bool grid_ok = __all_sync(kAll, tile_grid(m_tiles, num_tiles));
        int i = 0, out_box = 0;
        for (int tile = blockIdx.x; grid_ok && tile < num_tiles; tile += gridDim.x, ++i) {
            const int m_blk = tile % m_tiles;
            const int n_blk = tile / m_tiles;
            const int e = GROUPED ? expert_of_row(ind, E, m_blk * kTileM) : 0;
            const float alpha = GROUPED ? args.alpha[e] : alpha0;     // per expert in a grouped call
            const uint16_t* bias = (args.bias != nullptr) ? args.bias + (size_t)e * args.N : nullptr;
            if (!__all_sync(kAll, mbar_wait(tmem_full, i & 1, abort_flag))) break;
            tc_fence_after();
            uint32_t raw[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_load_32(tmem + lane_off + T::ACC + h * 128 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(raw + c * 32));
            tmem_load_wait();
            tc_fence_before();
            mbar_arrive(acc_empty);                    // the next tile's MMAs may start
            float v[128];
#pragma unroll
            for (int k = 0; k < 128; ++k) v[k] = __fmul_rn(alpha, __uint_as_float(raw[k]));
            if (MODE == Mode::Raw && lora_on) {
                // half 0 of the LoRA accumulator is complete with the base one (tmem_full); half 1
                // once lacc_full says so, after the h = 0 warps have released half 0
                if (h == 1 && !__all_sync(kAll, mbar_wait(lacc_full, i & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t lv[16];
                    tmem_load_16(tmem + lane_off + T::LACC + c * 16, lv);
                    tmem_load_wait();
#pragma unroll
                    for (int k = 0; k < 16; ++k) v[c * 16 + k] = __fmaf_rn(lora_s, __uint_as_float(lv[k]), v[c * 16 + k]);
                }
                tc_fence_before();
                mbar_arrive(lacc_empty);
            }
            const int row = m_blk * kTileM + rl;
            const int col0 = n_blk * kTileN + h * 128;
            if (bias != nullptr) {
                if (args.vec_out) {
                    // the producer put the tile's bias slice in shared memory (past N the values
                    // are stale, and those columns are clipped by the TMA store)
                    if (!__all_sync(kAll, mbar_wait(&bias_full[i & 1], (i >> 1) & 1, abort_flag))) break;
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
                            v[k] = __fadd_rn(v[k], __uint_as_float((uint32_t)__ldg(bias + col0 + k) << 16));
                }
            }
            if (args.vec_out) {
                // four 32 x 32 boxes per warp through kOutBoxes shared-memory buffers, each
                // written by a TMA store (rows past M and columns past N are clipped)
                uint8_t* box0 = smem + L::OUT_OFF + ew * kOutBoxes * L::OUT_BOX_BYTES;
                const int y0 = m_blk * kTileM + q * 32;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint8_t* box = box0 + out_box * L::OUT_BOX_BYTES;
                    if (++out_box == kOutBoxes) out_box = 0;
                    // the buffer's previous store (kOutBoxes stores back) has read it
                    if (lane == 0) bulk_wait_group_read<kOutBoxes - 1>();
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
                    if (lane == 0 && x < args.N && y0 < args.M) {
                        tma_store_2d(&tm_out, box, x, y0);
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
        // the TMA stores have finished reading shared memory and writing out before the CTA ends
        if (args.vec_out && lane == 0) bulk_wait_group_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, T::ALLOC);
    }
}

}  // namespace nvfp4lora
