// Decode-shaped NVFP4 x NVFP4 + LoRA GEMM (M <= 32 tokens), sm_100a.
//
// Same operation as gemm.cuh (flashinfer.gemm.mm_nvfp4_lora, opening formula; "Raw path" and
// "Prepared path" bullets), arranged for the case where the weights dominate the traffic:
//   * swapped operands: the MMA's 128-row side walks the weight rows n (b, b_sf, lora_b),
//     its N side holds the MT (16 or 32) token rows m (a, a_sf, d); the fp32 accumulator in
//     TMEM is out^T for one 128-column slice of out;
//   * split-K over a thread-block cluster: the S CTAs of a cluster each stream K/S of the
//     weights through a ring of stage slots (the whole split in flight at once where it fits).
//     Ranks 1..S-1 push their fp32 partials straight from registers into rank 0's shared memory
//     with st.async, each completing on a barrier of its own, and exit; rank 0 adds them in rank
//     order, each as soon as it has landed (so the result is deterministic), applies the epilogue
//     and the single bf16 rounding;
//   * rank 0 also computes the LoRA term, from buffers of its own: a second producer lane loads
//     its d and lora_b (or b_folded) chunks beside the base stages, and they are multiplied after
//     the base MMAs, into a TMEM region of their own on the raw path, into the base accumulator on
//     the prepared path (base first, LoRA after, alpha once);
//   * the raw combine is v = alpha*acc; v = fma(s, lacc, v); v += bias; the prepared combine is
//     v = alpha*acc (+ bias);
//   * before the dependency wait a CTA of a split plan warms L2 with what it will read (the small
//     activation-side tiles of a, a_sf and d, its weights and their scales), so that the loads
//     issued right after the wait meet fewer DRAM round trips.
// Zero-adapter path (Parameters: lora_scale): rank 0 reads the device scalar right after the
// dependency wait and issues no LoRA load or MMA when it is 0; it then combines exactly as the
// adapter-off instantiation does, so the output is bitwise the adapter-off output.
// The scale factors reach TMEM through the epilogue warps, which are idle until the accumulator
// is ready: a stage's scale atoms land on their own mbarrier (ahead of the large tiles), are read
// from shared memory and written with one tcgen05.st per warp in the layout a 32x128b.warpx4
// copy of the 128x4 atom produces, so the MMA thread only issues MMAs once the tiles are in.
// All waits are bounded; no global scratch memory is used.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace nvfp4lora {

struct DecodeArgs {
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const float* alpha;
    const float* scale;      // Raw: lora_scale; Prepared: ratio; Off: unused
    const uint16_t* lb;      // lora_b (raw) or b_folded (prepared): an L2 prefetch hint only
    const uint16_t* bias;
    uint16_t* out;
    int M, N, K, r;
    int n_tiles;             // ceil(N / 128)
    int splits;              // S: CTAs per cluster along K
    int stages_per_split;    // K / 256 / S
    int sf_atoms_k;          // K / 64
    int sf_row_blocks_b;     // ceil(N / 128)
    int pf_chunks;           // K chunks (256 wide) per L2-prefetch box
};

constexpr int kDecodeThreads = 192;       // producer, MMA, 4 epilogue warps

// STAGES ring slots; MAXS = the largest cluster split the plan leaves room for (rank 0 keeps
// MAXS - 1 peer partial slots).
template <int MT, int STAGES, int MAXS>
struct DecodeSmem {
    static constexpr int W_BYTES = 128 * 128;          // weight tile: 128 rows x 128 bytes
    static constexpr int X_BYTES = MT * 128;           // token tile: MT rows x 128 bytes
    static constexpr int SF_BYTES = 4 * 512;           // 4 scale atoms (one 128-row block)
    static constexpr int PART_SLOT = 128 * MT * 4;     // one peer's fp32 partial, [MT/4][128] float4
    static constexpr int LORA_CHUNKS = 2;              // r <= 128: two 64-wide chunks
    static constexpr int W_OFF = 0;
    static constexpr int X_OFF = W_OFF + STAGES * W_BYTES;
    static constexpr int SFW_OFF = X_OFF + STAGES * X_BYTES;
    static constexpr int SFX_OFF = SFW_OFF + STAGES * SF_BYTES;
    static constexpr int LW_OFF = SFX_OFF + STAGES * SF_BYTES;     // lora_b (or b_folded) chunks
    static constexpr int LX_OFF = LW_OFF + LORA_CHUNKS * W_BYTES;  // d chunks
    static constexpr int PART_OFF = LX_OFF + LORA_CHUNKS * X_BYTES;  // rank 0: peers' partials
    static constexpr int BAR_OFF = PART_OFF + (MAXS - 1) * PART_SLOT;
    // full[S], empty[S], sf_full[S], sf_ready[S], tmem_full, drain, lora_full, parts_full[MAXS - 1]
    static constexpr int NUM_BARS = 4 * STAGES + 3 + (MAXS - 1);
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int TOTAL = MISC_OFF + 16;
    static constexpr int DYN_BYTES = TOTAL + 1024;
    static_assert(X_BYTES % 1024 == 0, "token tiles must stay 1024-byte aligned");
    static_assert(DYN_BYTES <= 232448, "decode shared-memory plan exceeds 227 KB");
};

template <int MT, int STAGES>
struct DecodeTmem {
    static constexpr int ACC = 0;
    static constexpr int LACC = MT;
    static constexpr int SF0 = 2 * MT;
    static constexpr int SFW_COLS = 16;               // 4 MMAs x 4 columns (128 weight rows)
    static constexpr int SFX_COLS = 16;               // 4 MMAs x 4 columns (a padded 128-row atom)
    static constexpr int STAGE_COLS = SFW_COLS + SFX_COLS;
    static constexpr int USED = SF0 + STAGES * STAGE_COLS;
    static constexpr int ALLOC = USED <= 32 ? 32 : USED <= 64 ? 64 : USED <= 128 ? 128
                               : USED <= 256 ? 256 : 512;
    static_assert(USED <= 512, "decode TMEM plan exceeds 512 columns");
};

constexpr uint32_t kDecodeTmemBarrier = 2;   // named barrier: MMA warp + epilogue warps (160)
constexpr uint32_t kDecodeEpilogueBarrier = 3;   // named barrier: the 4 epilogue warps (128)
constexpr uint32_t kDecodeDeallocBarrier = 4;    // named barrier: MMA warp + epilogue warps (160)

template <int MT, int STAGES, int MAXS, Mode MODE>
__global__ void __launch_bounds__(kDecodeThreads, 1)
nvfp4_decode_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_lb,
                    const __grid_constant__ CUtensorMap tm_b3, const DecodeArgs args) {
    using L = DecodeSmem<MT, STAGES, MAXS>;
    using T = DecodeTmem<MT, STAGES>;
    static_assert(MT % 16 == 0 && MT <= 32, "MT must be 16 or 32");
    constexpr uint32_t IDESC_F4 = idesc_nvf4(MT);
    constexpr uint32_t IDESC_BF16 = idesc_bf16(MT);
    constexpr uint32_t kAll = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_full = empty + STAGES;   // the stage's scale atoms are in shared memory
    uint64_t* sf_ready = sf_full + STAGES;  // ... and in TMEM
    uint64_t* tmem_full = sf_ready + STAGES;
    uint64_t* drain = tmem_full + 1;
    uint64_t* lora_full = drain + 1;
    uint64_t* parts_full = lora_full + 1;   // rank 0: [p - 1] peer p's partial has landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    float* part = reinterpret_cast<float*>(smem + L::PART_OFF);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_blk = blockIdx.x;
    const int S = args.splits;
    const bool clustered = S > 1;
    const uint32_t rank = clustered ? cluster_rank() : 0u;
    const bool lora_rank = (MODE != Mode::Off) && rank == 0;   // computes the LoRA term
    const int k0 = (int)rank * args.stages_per_split;
    const int base_items = args.stages_per_split;
    const int lora_chunks = (args.r + 63) / 64;

    if (threadIdx.x == 0) {
        prefetch_tensor_map(&tm_b3);
        prefetch_tensor_map(&tm_b);
        prefetch_tensor_map(&tm_a);
        if (lora_rank) {
            prefetch_tensor_map(&tm_lb);
            prefetch_tensor_map(&tm_d);
        }
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_full[s], 1);
            mbar_init(&sf_ready[s], 4);
        }
        mbar_init(tmem_full, 1);
        mbar_init(drain, 1);
        mbar_init(lora_full, 1);
        for (int p = 0; p < MAXS - 1; ++p) mbar_init(&parts_full[p], 1);
        *abort_flag = 0;
        fence_mbar_init();
        // rank 0 expects each peer's [128][MT] fp32 partial on a barrier of its own (st.async bytes
        // may land before a barrier is waited on, never before it is armed: the peers wait on the
        // cluster barrier first)
        if (clustered && rank == 0)
            for (int p = 1; p < S; ++p) mbar_arrive_expect_tx(&parts_full[p - 1], (uint32_t)L::PART_SLOT);
    }
    __syncthreads();
    if (clustered) cluster_arrive();   // this CTA's barriers exist; waited on before remote access
    // Programmatic dependent launch: the next kernel on the stream may start its own prologue
    // now; every access to memory another kernel may write comes after grid_dependency_wait().
    grid_launch_dependents();

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            // A split plan warms L2 before the dependency wait (a prefetch changes no data and L2 is
            // where device memory is kept coherent, so it may precede the wait; the real loads come
            // after it): this CTA's K range of a and of a_sf's first 128-row block, on rank 0 the
            // d chunks and its lora_b rows, and its weights (one 3-D box covers up to 8 K chunks of
            // its 128 weight rows, whose scale atoms are contiguous).  Without a split the next
            // call's CTAs start on free SMs a whole call early, and warming then competed with this
            // call's own loads (M = 1, N = 14336, K = 4096, r = 8: 10.2 us per call with it, 8.9
            // without), so such a plan warms nothing.
            if (clustered) {
                for (int it = 0; it < base_items; ++it) tma_prefetch_l2_2d(&tm_a, (k0 + it) * 128, 0);
                bulk_prefetch_l2(args.a_sf + (size_t)k0 * 4 * 512, (uint32_t)min(base_items, 64) * 2048u);
                if (lora_rank) {
                    bulk_prefetch_l2(args.lb + (size_t)n_blk * 128 * args.r,
                                     (uint32_t)(min(128, args.N - n_blk * 128) * args.r * 2));
                    for (int c = 0; c < lora_chunks; ++c) tma_prefetch_l2_2d(&tm_d, c * 64, 0);
                }
                for (int c = 0; c < base_items; c += args.pf_chunks)
                    tma_prefetch_l2_3d(&tm_b3, 0, n_blk * 128, k0 + c);
                if (n_blk < args.sf_row_blocks_b)
                    bulk_prefetch_l2(args.b_sf + ((size_t)n_blk * args.sf_atoms_k + k0 * 4) * 512,
                                     (uint32_t)min(base_items, 64) * 2048u);
            }
            grid_dependency_wait();
            int stage = 0;
            uint32_t phase = 0, filled = 0, filled_parity = 0;
            bool ok = true;
            for (int it = 0; ok && it < base_items; ++it) {
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                const int kb = k0 + it;
                mbar_arrive_expect_tx(&sf_full[stage], 4096);
                bulk_load(smem + L::SFW_OFF + stage * L::SF_BYTES,
                          args.b_sf + ((size_t)n_blk * args.sf_atoms_k + kb * 4) * 512, 2048, &sf_full[stage]);
                bulk_load(smem + L::SFX_OFF + stage * L::SF_BYTES, args.a_sf + (size_t)kb * 4 * 512, 2048,
                          &sf_full[stage]);
                mbar_arrive_expect_tx(&full[stage], L::W_BYTES + L::X_BYTES);
                tma_load_2d(smem + L::W_OFF + stage * L::W_BYTES, &tm_b, &full[stage], kb * 128, n_blk * 128);
                tma_load_2d(smem + L::X_OFF + stage * L::X_BYTES, &tm_a, &full[stage], kb * 128, 0);
                filled |= 1u << stage;
                filled_parity = (filled_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok || *abort_flag) {
                for (int s = 0; s < STAGES; ++s)
                    if ((filled >> s) & 1u) {
                        mbar_wait(&sf_full[s], (filled_parity >> s) & 1u, nullptr);
                        mbar_wait(&full[s], (filled_parity >> s) & 1u, nullptr);
                    }
            }
        } else if (lane == 1 && lora_rank) {
            // The LoRA operands, issued by a lane of their own so that the zero-adapter decision
            // (a read of the device scalar after the dependency wait) holds up no base load: this
            // tile's 128 lora_b (b_folded) rows and the MT rows of d, 64 ranks per chunk, into
            // their own buffers.  A zero scale issues nothing.
            grid_dependency_wait();
            if (*args.scale != 0.0f) {
                mbar_arrive_expect_tx(lora_full, lora_chunks * (L::W_BYTES + L::X_BYTES));
                for (int c = 0; c < lora_chunks; ++c) {
                    tma_load_2d(smem + L::LW_OFF + c * L::W_BYTES, &tm_lb, lora_full, c * 64, n_blk * 128);
                    tma_load_2d(smem + L::LX_OFF + c * L::X_BYTES, &tm_d, lora_full, c * 64, 0);
                }
                // the LoRA bytes land before the CTA can end
                mbar_wait(lora_full, 0, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        tmem_alloc(tmem_slot, T::ALLOC);
        tmem_relinquish();
        tc_fence_before();
        named_barrier_sync(kDecodeTmemBarrier, 160);   // hands the TMEM address to the epilogue
        tc_fence_after();
        const uint32_t tmem = *tmem_slot;
        if (lane == 0) {
            grid_dependency_wait();
            float sv = 0.0f;
            if (lora_rank) sv = *args.scale;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int it = 0; ok && it < base_items; ++it) {
                if (!mbar_wait(&sf_ready[stage], phase, abort_flag)) { ok = false; break; }
                if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t w_addr = smem_u32(smem + L::W_OFF + stage * L::W_BYTES);
                const uint32_t x_addr = smem_u32(smem + L::X_OFF + stage * L::X_BYTES);
                const uint32_t sfw_t = tmem + T::SF0 + stage * T::STAGE_COLS;
                const uint32_t sfx_t = sfw_t + T::SFW_COLS;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tc_mma_nvf4(tmem + T::ACC, sdesc_sw128(w_addr + j * 32), sdesc_sw128(x_addr + j * 32),
                                IDESC_F4, sfw_t + 4 * j, sfx_t + 4 * j, (it > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (ok && lora_rank && sv != 0.0f) {
                // raw: its own accumulator; prepared: the base accumulator, after the base product
                if (!mbar_wait(lora_full, 0, abort_flag)) ok = false;
                if (ok) {
                    tc_fence_after();
                    const uint32_t dst = tmem + ((MODE == Mode::Prepared) ? T::ACC : T::LACC);
                    for (int c = 0; c < lora_chunks; ++c) {
                        const uint32_t w_addr = smem_u32(smem + L::LW_OFF + c * L::W_BYTES);
                        const uint32_t x_addr = smem_u32(smem + L::LX_OFF + c * L::X_BYTES);
                        const int rem = args.r - c * 64;
                        const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                        for (int j = 0; j < ksteps; ++j)
                            tc_mma_bf16(dst, sdesc_sw128(w_addr + j * 32), sdesc_sw128(x_addr + j * 32), IDESC_BF16,
                                        (MODE == Mode::Prepared || c > 0 || j > 0) ? 1u : 0u);
                    }
                }
            }
            if (ok) tc_commit(tmem_full);
            if (!ok || *abort_flag) {
                tc_commit(drain);
                mbar_wait(drain, 0, nullptr);
            }
        }
        __syncwarp();
        // TMEM goes back as soon as the epilogue warps hold the accumulators in registers
        named_barrier_sync(kDecodeDeallocBarrier, 160);
        tc_fence_after();
        tmem_dealloc(tmem, T::ALLOC);
    } else {
        // ------------------------------- epilogue -----------------------------------
        const int q = warp & 3;
        const int nl = q * 32 + lane;                 // weight row within the tile = TMEM lane
        const int n = n_blk * 128 + nl;               // output column
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        grid_dependency_wait();
        // only rank 0 combines: it reads the scalars and its bias element (consumed at the end)
        float lora_s = 0.0f;
        if (MODE != Mode::Off && rank == 0) lora_s = *args.scale;
        const bool lora_on = (lora_s != 0.0f);        // false on ranks > 0
        const float alpha = (rank == 0) ? *args.alpha : 0.0f;
        const float bias_v = (rank == 0 && args.bias != nullptr && n < args.N)
                                 ? __uint_as_float((uint32_t)__ldg(args.bias + n) << 16) : 0.0f;
        named_barrier_sync(kDecodeTmemBarrier, 160);
        tc_fence_after();
        const uint32_t tmem = *tmem_slot;
        bool ok = true;
        // every peer's barriers exist before any remote access; waited here, off the critical path
        if (clustered) cluster_wait();
        {
            // stage each base stage's scale factors into TMEM once its atoms have landed: columns
            // [4j, 4j+4) take weight-scale atom j, [16+4j, 16+4j+4) token-scale atom j; lane l of
            // every lane quarter holds atom row l (the 32x128b.warpx4 layout)
            int stage = 0;
            uint32_t phase = 0;
            for (int it = 0; ok && it < base_items; ++it) {
                ok = __all_sync(kAll, mbar_wait(&sf_full[stage], phase, abort_flag));
                if (!ok) break;
                const uint8_t* sfw = smem + L::SFW_OFF + stage * L::SF_BYTES + lane * 16;
                const uint8_t* sfx = smem + L::SFX_OFF + stage * L::SF_BYTES + lane * 16;
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 w = *reinterpret_cast<const uint4*>(sfw + j * 512);
                    const uint4 x = *reinterpret_cast<const uint4*>(sfx + j * 512);
                    v[4 * j] = w.x; v[4 * j + 1] = w.y; v[4 * j + 2] = w.z; v[4 * j + 3] = w.w;
                    v[16 + 4 * j] = x.x; v[16 + 4 * j + 1] = x.y; v[16 + 4 * j + 2] = x.z; v[16 + 4 * j + 3] = x.w;
                }
                tmem_store_32(tmem + lane_off + T::SF0 + stage * T::STAGE_COLS, v);
                tmem_store_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
        if (ok) ok = __all_sync(kAll, mbar_wait(tmem_full, 0, abort_flag));
        float acc[MT], lac[MT];
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < MT / 16; ++c) {
                uint32_t v[16];
                tmem_load_16(tmem + lane_off + T::ACC + c * 16, v);
                tmem_load_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[c * 16 + i] = __uint_as_float(v[i]);
            }
            if (MODE == Mode::Raw && lora_on) {
#pragma unroll
                for (int c = 0; c < MT / 16; ++c) {
                    uint32_t v[16];
                    tmem_load_16(tmem + lane_off + T::LACC + c * 16, v);
                    tmem_load_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) lac[c * 16 + i] = __uint_as_float(v[i]);
                }
            }
        }
        tc_fence_before();
        named_barrier_arrive(kDecodeDeallocBarrier, 160);   // accumulators read: TMEM may go
        // a peer's partial slot is [MT/4][128] float4: lane-consecutive 16-byte accesses
        if (rank != 0) {
            // push the partial into rank 0's slot (rank - 1); the bytes complete on its barrier
            if (ok) {
                const uint32_t dst = map_to_rank(smem_u32(part + (size_t)(rank - 1) * 128 * MT + nl * 4), 0);
                const uint32_t bar = map_to_rank(smem_u32(&parts_full[rank - 1]), 0);
#pragma unroll
                for (int m = 0; m < MT; m += 4)
                    st_async_v4(dst + m * 128 * 4, acc[m], acc[m + 1], acc[m + 2], acc[m + 3], bar);
            }
        } else {
            // the peers' partials in rank order, each as soon as it has landed
            int seen = 1;                              // ranks whose partial has been added
            if (ok) {
                for (int pr = 1; pr < S; ++pr) {
                    ok = __all_sync(kAll, mbar_wait_cluster(&parts_full[pr - 1], 0, abort_flag));
                    if (!ok) break;
                    const float4* src = reinterpret_cast<const float4*>(part + (size_t)(pr - 1) * 128 * MT) + nl;
#pragma unroll
                    for (int m = 0; m < MT; m += 4) {
                        const float4 w = src[(m / 4) * 128];
                        acc[m] = __fadd_rn(acc[m], w.x);
                        acc[m + 1] = __fadd_rn(acc[m + 1], w.y);
                        acc[m + 2] = __fadd_rn(acc[m + 2], w.z);
                        acc[m + 3] = __fadd_rn(acc[m + 3], w.w);
                    }
                    seen = pr + 1;
                }
            }
            // out^T slice -> bf16 tile [MT][128] in the first weight slot (every MMA that read it
            // has completed), then 16-byte row stores
            uint16_t* tile = reinterpret_cast<uint16_t*>(smem + L::W_OFF);
            if (ok) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float x = __fmul_rn(alpha, acc[m]);
                    if (MODE == Mode::Raw && lora_on) x = __fmaf_rn(lora_s, lac[m], x);
                    if (args.bias != nullptr) x = __fadd_rn(x, bias_v);
                    tile[m * 128 + nl] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
                }
            }
            named_barrier_sync(kDecodeEpilogueBarrier, 128);
            if (ok) {
                const bool vec = (args.N % 8) == 0;    // rows of out are 16-byte aligned
#pragma unroll
                for (int i = 0; i < MT * 16 / 128; ++i) {
                    const int chunk = threadIdx.x - 64 + i * 128;
                    const int m = chunk >> 4, c8 = chunk & 15;
                    const int n0 = n_blk * 128 + c8 * 8;
                    if (m >= args.M || n0 >= args.N) continue;
                    const uint16_t* src = tile + m * 128 + c8 * 8;
                    uint16_t* dst = args.out + (size_t)m * args.N + n0;
                    if (vec && n0 + 8 <= args.N) {
                        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
                    } else {
                        for (int e = 0; e < 8 && n0 + e < args.N; ++e) dst[e] = src[e];
                    }
                }
            }
            // rank 0 stays until every peer's bytes have landed (also after an error: bounded
            // waits), so no remote store reaches shared memory that was handed on
            for (int pr = seen; pr < S; ++pr) mbar_wait_cluster(&parts_full[pr - 1], 0, nullptr);
        }
    }
    // Every thread arrived on the cluster barrier once; the ones that did not need it wait here,
    // so each thread completes exactly one arrive/wait pair.
    if (clustered && warp < 2) cluster_wait();
}

}  // namespace nvfp4lora
