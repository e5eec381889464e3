// The routed-MoE FC2 (down projection) LoRA delta (flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta,
// opening formula and Parameters):
//     delta[t] = scale * sum_j w[t, j] * ( B_down[l, e] @ ( A_down[l, e] @ act[p] ) )
// for token t with adapter l = lora_ids[t] (negative: no adapter, delta 0) and routed slots j
// (expert e = topk_ids[t, j], weight w = topk_weights[t, j], activation row p = the slot's
// permuted index, negative: inactive slot).  A_down[l, e] is the [rank, I] row-major block
// l * stride_a elements into expert e's A bank, B_down[l, e] the [H, rank] row-major block
// l * stride_b elements into its B bank; the activation and the banks hold bf16 or fp16 values.
//
// One thread-block cluster of CS CTAs per token.  CTA c of the cluster
//   1. shrink: forms partial sums v_c[j][k] = sum over its slice of the I columns of
//      A[k, i] * act[p_j, i] in fp32, for every active slot j and k < rank;
//   2. exchange: stores its partials into slot c of every CTA's gather buffer (distributed shared
//      memory); after one cluster barrier each CTA adds the CS partials in rank order, so all of
//      them hold the same v and the order of the sum is fixed;
//   3. expand: for its slice of the H output columns,
//      out[t, h] = round(scale * sum_j w_j * sum_k B_j[h, k] * v[j][k]).
// The work is a gather of small matrix-vector products, memory-bound: each CTA streams its column
// slices of A and row slices of B with 16-byte read-only loads; the B slices are prefetched into L2
// as soon as the routing is read, so the expand finds them there after the shrink and exchange.
// A routing entry that cannot be honoured (expert id out of range, activation row past the
// buffer, a bank address that is null or not 16-byte aligned) is skipped and reported through
// the device error word; no out-of-range address is dereferenced.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "fold.cuh"
#include "ptx.cuh"

namespace nvfp4lora {

constexpr int kBgmvThreads = 256;
constexpr int kBgmvMaxTopK = 16;
constexpr int kBgmvMaxRank = 128;
constexpr int kBgmvMaxCluster = 8;
constexpr int kErrBadRoute = 3;         // device error word: a routing entry was out of range
constexpr int kBgmvSmemLimit = 200 * 1024;   // dynamic shared memory of one CTA, bytes

struct BgmvArgs {
    const void* act;            // [rows, I] lora dtype
    const int32_t* perm;        // [T * top_k] expanded index -> permuted row
    const int64_t* w_ptr_a;     // [num_experts] A bank addresses
    const int64_t* w_ptr_b;     // [num_experts] B bank addresses
    const int32_t* topk_ids;    // [T, top_k]
    const float* topk_w;        // [T, top_k]
    const int32_t* lora_ids;    // [T]
    void* out;                  // [T, H] out dtype
    int64_t stride_a;           // elements between adapters in an A bank
    int64_t stride_b;           // elements between adapters in a B bank
    int rows, I, top_k, num_experts, rank, H, cs;
    float scale;
};

struct BgmvSlot {
    const uint4* a;             // A_down[l, e], row-major [rank][I / 8] vectors
    const uint4* b;             // B_down[l, e], row-major [H][rank / 8] vectors
    const uint4* x;             // the slot's activation row, I / 8 vectors
    float w;
    int active;
};

// Eight packed 16-bit values (one 16-byte vector) as fp32 pairs; both conversions are exact.
template <bool F16>
__device__ __forceinline__ float2 unpack_pair(uint32_t u) {
    if constexpr (F16) {
        __half2 h;
        memcpy(&h, &u, 4);
        return __half22float2(h);
    } else {
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
}

template <bool F16>
__device__ __forceinline__ float dot8(float acc, const uint4& a, const uint4& x) {
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 fa = unpack_pair<F16>(aw[q]);
        const float2 fx = unpack_pair<F16>(xw[q]);
        acc = fmaf(fa.x, fx.x, acc);
        acc = fmaf(fa.y, fx.y, acc);
    }
    return acc;
}

template <bool F16>
__device__ __forceinline__ float dot8_smem(float acc, const uint4& a, const float* v) {
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 fa = unpack_pair<F16>(aw[q]);
        acc = fmaf(fa.x, v[2 * q], acc);
        acc = fmaf(fa.y, v[2 * q + 1], acc);
    }
    return acc;
}

// Read-only 16-byte loads: `ld_keep` for the activation row, which every k of a slot reads again
// (kept in L1), `ld_stream` for bank data read once per CTA.
__device__ __forceinline__ uint4 ld_keep(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Plain 16-byte store into the shared memory of a CTA of this cluster (address from map_to_rank);
// the cluster barrier that follows makes it visible to that CTA.
__device__ __forceinline__ void st_cluster_v4(uint32_t caddr, const float4& v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"r"(caddr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

// Shared memory of one CTA, in floats: the partials (len), the shrink's cells (len x chunks of 32
// vectors of the CTA's I slice), the gather buffer (cs x len) and the sum (len).  The gather has a
// region of its own: peers write into it while this CTA may still be adding up its cells.
__host__ __device__ constexpr int64_t bgmv_smem_floats(int64_t len, int64_t slice_vectors, int64_t cs) {
    return len * (2 + cs + (slice_vectors + 31) / 32);
}

template <bool F16_OUT>
__device__ __forceinline__ void store_out(void* out, int64_t idx, float y) {
    if constexpr (F16_OUT) {
        static_cast<__half*>(out)[idx] = __float2half_rn(y);
    } else {
        static_cast<uint16_t*>(out)[idx] = (uint16_t)f32_to_bf16_bits(y);
    }
}

// Launch: grid T * cs CTAs of kBgmvThreads, clusters of cs along x (cs = 1: no cluster);
// dynamic shared memory bgmv_smem_floats(...) floats.
template <bool F16_IN, bool F16_OUT>
__global__ void __launch_bounds__(kBgmvThreads, 4)
bgmv_delta_kernel(const BgmvArgs args) {
    extern __shared__ __align__(16) float bgmv_smem[];
    __shared__ BgmvSlot slots[kBgmvMaxTopK];
    __shared__ int s_lid;

    const int cs = args.cs;
    const int c = cs > 1 ? (int)cluster_rank() : 0;
    const int t = blockIdx.x / cs;
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    const int top_k = args.top_k, rank = args.rank;
    const int len = top_k * rank;
    const int h0 = (int)((int64_t)args.H * c / cs);
    const int h1 = (int)((int64_t)args.H * (c + 1) / cs);

    grid_dependency_wait();
    grid_launch_dependents();

    // ---- routing: the token's adapter and its slots, read in one round of loads ----
    if (tid < top_k) {
        BgmvSlot s{nullptr, nullptr, nullptr, 0.0f, 0};
        const int64_t x = (int64_t)t * top_k + tid;
        const int lid = args.lora_ids[t];
        const int p = args.perm[x];
        const int e = args.topk_ids[x];
        const float wt = args.topk_w[x];
        if (tid == 0) s_lid = lid;
        if (lid >= 0 && p >= 0) {
            bool ok = p < args.rows && e >= 0 && e < args.num_experts;
            uintptr_t pa = 0, pb = 0;
            if (ok) {
                const int64_t ba = args.w_ptr_a[e], bb = args.w_ptr_b[e];
                pa = (uintptr_t)ba + (uintptr_t)((int64_t)lid * args.stride_a * 2);
                pb = (uintptr_t)bb + (uintptr_t)((int64_t)lid * args.stride_b * 2);
                ok = ba != 0 && bb != 0 && ((pa | pb) & 15u) == 0;
            }
            if (ok) {
                s.a = reinterpret_cast<const uint4*>(pa);
                s.b = reinterpret_cast<const uint4*>(pb);
                s.x = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(args.act) + (int64_t)p * args.I);
                s.w = wt;
                s.active = 1;
                // this CTA's B rows [h0, h1) are contiguous: pull them into L2 for the expand
                if (h1 > h0) bulk_prefetch_l2(s.b + (int64_t)h0 * (rank / 8), (uint32_t)((h1 - h0) * rank * 2));
            } else {
                atomicExch(&g_device_error, kErrBadRoute);
            }
        }
        slots[tid] = s;
    }
    __syncthreads();
    if (s_lid < 0) {
        // no adapter: a zero delta; the whole cluster takes this branch and reaches no barrier
        for (int h = h0 + tid; h < h1; h += kBgmvThreads) store_out<F16_OUT>(args.out, (int64_t)t * args.H + h, 0.0f);
        return;
    }

    // ---- shrink: partial v over this CTA's slice of the I columns ----
    // Work unit = (slot j, chunk of 32 vectors of the slice, group of 4 rows of A_j): a lane loads
    // one activation vector and the 4 matching A vectors.  A warp takes 2 units at a time and
    // issues their 10 loads before the first multiply.  Each unit's 4 sums go to their own cells,
    // and the cells of a row are added in chunk order, so the result does not depend on the schedule.
    float* part = bgmv_smem;                           // [len]
    float* cells = part + len;                         // [len][nch]
    const int nv = args.I / 8;
    const int v0 = (int)((int64_t)nv * c / cs), v1 = (int)((int64_t)nv * (c + 1) / cs);
    const int nch = (v1 - v0 + 31) / 32;
    const int kq = rank / 4;
    const int units = top_k * nch * kq;
    for (int u0 = warp * 2; u0 < units; u0 += (kBgmvThreads / 32) * 2) {
        uint4 av[2][4], xv[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int u = u0 + q;
            const int j = u / (nch * kq), ch = (u / kq) % nch, k0 = (u % kq) * 4;
            const int vi = v0 + ch * 32 + lane;
            const bool on = u < units && vi < v1 && slots[j < top_k ? j : 0].active;
            const BgmvSlot& s = slots[j < top_k ? j : 0];
            xv[q] = on ? ld_keep(s.x + vi) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < 4; ++r)
                av[q][r] = on ? ld_stream(s.a + (int64_t)(k0 + r) * nv + vi) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int u = u0 + q;
            const int j = u / (nch * kq), ch = (u / kq) % nch, k0 = (u % kq) * 4;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float acc = dot8<F16_IN>(0.0f, av[q][r], xv[q]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
                if (lane == 0 && u < units) cells[(j * rank + k0 + r) * nch + ch] = acc;
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < len; i += kBgmvThreads) {
        float sum = cells[i * nch];
        for (int k = 1; k < nch; ++k) sum += cells[i * nch + k];
        part[i] = sum;
    }
    __syncthreads();

    // ---- exchange: every CTA gets the CS partials, adds them in rank order ----
    const float* v = part;
    if (cs > 1) {
        // the same offset in every CTA of the cluster: sized by the largest slice, not this CTA's
        const int nch_max = ((nv + cs - 1) / cs + 31) / 32;
        float* gather = cells + len * nch_max;      // [cs][len], written by every CTA of the cluster
        float* vsum = gather + cs * len;            // [len]
        for (int i = tid; i < len / 4; i += kBgmvThreads) {
            const float4 val = reinterpret_cast<const float4*>(part)[i];
            const uint32_t local = smem_u32(gather + c * len + 4 * i);
            for (int q = 0; q < cs; ++q) st_cluster_v4(map_to_rank(local, (uint32_t)q), val);
        }
        cluster_arrive();
        cluster_wait();
        // no CTA touches another's shared memory after the barrier, so any CTA may exit after it
        for (int i = tid; i < len; i += kBgmvThreads) {
            float sum = gather[i];
            for (int q = 1; q < cs; ++q) sum += gather[q * len + i];
            vsum[i] = sum;
        }
        __syncthreads();
        v = vsum;
    }

    // ---- expand: this CTA's output columns [h0, h1), two rows per thread at a time; the loads of
    // 2 slots x 2 vectors of both rows are issued before the first multiply ----
    const int rv = rank / 8;
    for (int ha = h0 + tid; ha < h1; ha += 2 * kBgmvThreads) {
        const int hb = ha + kBgmvThreads;
        const bool has_b = hb < h1;
        float acc_a = 0.0f, acc_b = 0.0f;
        for (int j0 = 0; j0 < top_k; j0 += 2) {
            float ua[2] = {0.0f, 0.0f}, ub[2] = {0.0f, 0.0f};
            for (int q0 = 0; q0 < rv; q0 += 2) {
                uint4 ba[2][2], bb[2][2];
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int j = j0 + jj;
                    const bool on = j < top_k && slots[j].active;
                    const uint4* base = on ? slots[j].b : nullptr;
#pragma unroll
                    for (int qq = 0; qq < 2; ++qq) {
                        const bool vq = on && q0 + qq < rv;
                        ba[jj][qq] = vq ? ld_stream(base + (int64_t)ha * rv + q0 + qq) : make_uint4(0, 0, 0, 0);
                        bb[jj][qq] = vq && has_b ? ld_stream(base + (int64_t)hb * rv + q0 + qq) : make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int j = j0 + jj;
                    if (j < top_k) {
                        const float* vj = v + j * rank + 8 * q0;
#pragma unroll
                        for (int qq = 0; qq < 2; ++qq) {
                            if (q0 + qq < rv) {
                                ua[jj] = dot8_smem<F16_IN>(ua[jj], ba[jj][qq], vj + 8 * qq);
                                ub[jj] = dot8_smem<F16_IN>(ub[jj], bb[jj][qq], vj + 8 * qq);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = j0 + jj;
                if (j < top_k && slots[j].active) {
                    acc_a = fmaf(slots[j].w, ua[jj], acc_a);
                    acc_b = fmaf(slots[j].w, ub[jj], acc_b);
                }
            }
        }
        store_out<F16_OUT>(args.out, (int64_t)t * args.H + ha, args.scale * acc_a);
        if (has_b) store_out<F16_OUT>(args.out, (int64_t)t * args.H + hb, args.scale * acc_b);
    }
}

}  // namespace nvfp4lora
