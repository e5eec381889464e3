// Decode-shaped NVFP4 x NVFP4 + LoRA GEMM (M <= 32 tokens), sm_100a.
//
// Same operation as gemm.cuh (flashinfer.gemm.mm_nvfp4_lora, opening formula; "Raw path" and
// "Prepared path" bullets), arranged for the case where the weights dominate the traffic:
//   * swapped operands: the MMA's 128-row side walks the weight rows n (b, b_sf, lora_b),
//     its N side holds the MT (16 or 32) token rows m (a, a_sf, d); the fp32 accumulator in
//     TMEM is out^T for one 128-column slice of out;
//   * split-K over a thread-block cluster: the S CTAs of a cluster each stream K/S of the
//     weights.  Ranks 1..S-1 push their fp32 partials straight from registers into rank 0's
//     shared memory with st.async, whose bytes complete on rank 0's pre-armed mbarrier (one
//     one-way trip), and exit; rank 0 sums them in rank order (so the result is
//     deterministic), adds the LoRA term it computed into its own TMEM region, applies the
//     epilogue and the single bf16 rounding;
//   * the raw combine is v = alpha*acc; v = fma(s, lacc, v); v += bias; the prepared combine
//     adds the folded LoRA term to the fully reduced base accumulator, then v = alpha*acc
//     (+ bias) -- base first, LoRA after, alpha once.
// The producer issues the whole first fill of the stage ring right after the dependency wait, and
// the LoRA operands (own buffers) right after it.  The scale factors reach TMEM through the
// epilogue warps, which are idle until the accumulator is ready: a stage's scale atoms land on
// their own mbarrier (ahead of the large tiles), are read from shared memory and written with
// one tcgen05.st per warp in the layout a 32x128b.warpx4 copy of the 128x4 atom produces, so
// the MMA thread only issues MMAs once the tiles are in.
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

// MAXS = the largest cluster split the plan leaves room for (rank 0 keeps MAXS - 1 partial slots).
template <int MT, int STAGES, int MAXS>
struct DecodeSmem {
    static constexpr int W_BYTES = 128 * 128;          // weight tile: 128 rows x 128 bytes
    static constexpr int X_BYTES = MT * 128;           // token tile: MT rows x 128 bytes
    static constexpr int SF_BYTES = 4 * 512;           // 4 scale atoms (one 128-row block)
    static constexpr int PART_SLOT = 128 * MT * 4;     // one peer's fp32 partial, [MT/4][128] float4
    static constexpr int W_OFF = 0;
    static constexpr int X_OFF = W_OFF + STAGES * W_BYTES;
    static constexpr int SFW_OFF = X_OFF + STAGES * X_BYTES;
    static constexpr int SFX_OFF = SFW_OFF + STAGES * SF_BYTES;
    static constexpr int LORA_CHUNKS = 2;              // r <= 128: two 64-wide chunks
    static constexpr int LW_OFF = SFX_OFF + STAGES * SF_BYTES;     // lora_b (or b_folded) chunks
    static constexpr int LX_OFF = LW_OFF + LORA_CHUNKS * W_BYTES;  // d chunks
    static constexpr int PART_OFF = LX_OFF + LORA_CHUNKS * X_BYTES;  // rank 0: peers' partials
    static constexpr int BAR_OFF = PART_OFF + (MAXS - 1) * PART_SLOT;
    // full[S], empty[S], sf_full[S], sf_ready[S], tmem_full, drain, parts_full, lora_full
    static constexpr int NUM_BARS = 4 * STAGES + 4;
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
    static_assert(USED <= 512, "TMEM plan exceeds 512 columns");
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

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_full = empty + STAGES;   // the stage's scale atoms are in shared memory
    uint64_t* sf_ready = sf_full + STAGES;  // ... and in TMEM
    uint64_t* tmem_full = sf_ready + STAGES;
    uint64_t* drain = tmem_full + 1;
    uint64_t* parts_full = drain + 1;    // rank 0: every peer's partial has landed
    uint64_t* lora_full = parts_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    float* part = reinterpret_cast<float*>(smem + L::PART_OFF);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_blk = blockIdx.x;
    const bool clustered = args.splits > 1;
    const uint32_t rank = clustered ? cluster_rank() : 0u;
    const int k0 = (int)rank * args.stages_per_split;
    const int base_items = args.stages_per_split;

    // The zero-adapter decision (rank 0 only) reads a device scalar; each role issues the load
    // early and consumes it once its base work is under way.
    auto lora_scale_value = [&]() -> float {
        if constexpr (MODE != Mode::Off) return rank == 0 ? *args.scale : 0.0f;
        return 0.0f;
    };

    if (threadIdx.x == 0) {
        prefetch_tensor_map(&tm_b3);
        prefetch_tensor_map(&tm_b);
        prefetch_tensor_map(&tm_a);
        if (MODE != Mode::Off && rank == 0) {
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
        mbar_init(parts_full, 1);
        mbar_init(lora_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // rank 0 expects every peer's [128][MT] fp32 partial (st.async bytes may land first)
        if (clustered && rank == 0) mbar_arrive_expect_tx(parts_full, (uint32_t)(args.splits - 1) * L::PART_SLOT);
    }
    __syncthreads();
    if (clustered) cluster_arrive();   // this CTA's barriers exist; waited on before remote access
    // Programmatic dependent launch: the next kernel on the stream may start its own prologue
    // now; every access to memory another kernel may write comes after grid_dependency_wait().
    grid_launch_dependents();

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            // Warm L2 with this CTA's weight tiles while the previous kernel finishes (a prefetch
            // changes no data, so it may precede the dependency wait): one 3-D box covers the
            // CTA's whole K range of its 128 weight rows, and their scale atoms are contiguous.
            for (int c = 0; c < base_items; c += args.pf_chunks)
                tma_prefetch_l2_3d(&tm_b3, 0, n_blk * 128, k0 + c);
            if (n_blk < args.sf_row_blocks_b)
                bulk_prefetch_l2(args.b_sf + ((size_t)n_blk * args.sf_atoms_k + k0 * 4) * 512,
                                 (uint32_t)min(base_items, 64) * 2048u);
            // rank 0 computes the LoRA term: its 128 rows of lora_b / b_folded are contiguous
            if (MODE != Mode::Off && rank == 0)
                bulk_prefetch_l2(args.lb + (size_t)n_blk * 128 * args.r,
                                 (uint32_t)(min(128, args.N - n_blk * 128) * args.r * 2));
            grid_dependency_wait();
            int stage = 0;
            uint32_t phase = 0, filled = 0, filled_parity = 0;
            bool ok = true, lora_issued = false;
            auto next_stage = [&]() {
                filled |= 1u << stage;
                filled_parity = (filled_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            };
            if (MODE != Mode::Off && rank == 0) {
                // The LoRA operands first, into their own buffers: they were warmed into L2 before
                // the dependency wait, so they land before the base tiles.  A zero scale (read
                // later) skips the LoRA MMAs; only these reads remain.
                const int chunks = (args.r + 63) / 64;
                mbar_arrive_expect_tx(lora_full, chunks * (L::W_BYTES + L::X_BYTES));
                for (int c = 0; c < chunks; ++c) {
                    tma_load_2d(smem + L::LW_OFF + c * L::W_BYTES, &tm_lb, lora_full, c * 64, n_blk * 128);
                    tma_load_2d(smem + L::LX_OFF + c * L::X_BYTES, &tm_d, lora_full, c * 64, 0);
                }
                lora_issued = true;
            }
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
                next_stage();
            }
            if (!ok || *abort_flag) {
                for (int s = 0; s < STAGES; ++s)
                    if ((filled >> s) & 1u) {
                        mbar_wait(&sf_full[s], (filled_parity >> s) & 1u, nullptr);
                        mbar_wait(&full[s], (filled_parity >> s) & 1u, nullptr);
                    }
            }
            // the LoRA bytes land before the CTA can end, also when a zero scale skipped their MMAs
            if (lora_issued) mbar_wait(lora_full, 0, nullptr);
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
            const float sv = (rank == 0) ? lora_scale_value() : 0.0f;
            bool ok = true;
            if (sv != 0.0f) {
                // the LoRA operands were issued first and land first: their MMAs go first
                if (!mbar_wait(lora_full, 0, abort_flag)) ok = false;
                if (ok) {
                    tc_fence_after();
                    const int chunks = (args.r + 63) / 64;
                    for (int c = 0; c < chunks; ++c) {
                        const uint32_t w_addr = smem_u32(smem + L::LW_OFF + c * L::W_BYTES);
                        const uint32_t x_addr = smem_u32(smem + L::LX_OFF + c * L::X_BYTES);
                        const int rem = args.r - c * 64;
                        const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
                        for (int j = 0; j < ksteps; ++j)
                            tc_mma_bf16(tmem + T::LACC, sdesc_sw128(w_addr + j * 32), sdesc_sw128(x_addr + j * 32),
                                        IDESC_BF16, (c > 0 || j > 0) ? 1u : 0u);
                    }
                }
            }
            int stage = 0;
            uint32_t phase = 0;
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
        const float lora_s = lora_scale_value();
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
                ok = __all_sync(0xffffffffu, mbar_wait(&sf_full[stage], phase, abort_flag));
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
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(tmem_full, 0, abort_flag));
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
            if (lora_on) {
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
        bool parts_seen = false;
        // a peer's partial slot is [MT/4][128] float4: lane-consecutive 16-byte accesses
        if (rank != 0) {
            // push the partial into rank 0's slot (rank - 1); the bytes complete on its barrier
            if (ok) {
                const uint32_t dst = map_to_rank(smem_u32(part + (size_t)(rank - 1) * 128 * MT + nl * 4), 0);
                const uint32_t bar = map_to_rank(smem_u32(parts_full), 0);
#pragma unroll
                for (int m = 0; m < MT; m += 4)
                    st_async_v4(dst + m * 128 * 4, acc[m], acc[m + 1], acc[m + 2], acc[m + 3], bar);
            }
        } else {
            if (ok && clustered) {
                ok = __all_sync(0xffffffffu, mbar_wait_cluster(parts_full, 0, abort_flag));
                parts_seen = ok;
                if (ok) {
                    for (int pr = 1; pr < args.splits; ++pr) {
                        const float4* src = reinterpret_cast<const float4*>(part + (size_t)(pr - 1) * 128 * MT) + nl;
#pragma unroll
                        for (int m = 0; m < MT; m += 4) {
                            const float4 w = src[(m / 4) * 128];
                            acc[m] = __fadd_rn(acc[m], w.x);
                            acc[m + 1] = __fadd_rn(acc[m + 1], w.y);
                            acc[m + 2] = __fadd_rn(acc[m + 2], w.z);
                            acc[m + 3] = __fadd_rn(acc[m + 3], w.w);
                        }
                    }
                }
            }
            // out^T slice -> bf16 tile [MT][128] in the first weight stage (every MMA that read it
            // has completed), then 16-byte row stores
            uint16_t* tile = reinterpret_cast<uint16_t*>(smem + L::W_OFF);
            if (ok) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float a = acc[m];
                    if (MODE == Mode::Prepared && lora_on) a = __fadd_rn(a, lac[m]);
                    float x = __fmul_rn(alpha, a);
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
        }
        // rank 0 stays until every peer's bytes have landed (also after an error: a bounded wait),
        // so no remote store reaches shared memory that was handed on
        if (clustered && rank == 0 && !parts_seen) mbar_wait_cluster(parts_full, 0, nullptr);
    }
    // Every thread arrived on the cluster barrier once; the ones that did not need it wait here,
    // so each thread completes exactly one arrive/wait pair.
    if (clustered && warp < 2) cluster_wait();
}

}  // namespace nvfp4lora
