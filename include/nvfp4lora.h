/*
 * nvfp4lora -- NVFP4 block-scaled GEMM with a fused BF16 LoRA correction, for B200
 * (sm_100a).  C ABI.
 *
 * The operation (flashinfer.gemm.mm_nvfp4_lora, opening formula):
 *
 *     out = bf16_rne( alpha * (dequant(a) @ dequant(b)^T)
 *                     + lora_scale * (d @ lora_b^T) [+ bias] )
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer on the current CUDA device, except the
 *     adapter structs, which live in host memory.  The caller owns all device memory
 *     (inputs, out, b_folded, ratio); the library never allocates device memory.
 *   - bf16 tensors are passed as uint16_t bit patterns; fp32 scalars as one-element
 *     device arrays (graph-capturable: read by the kernels at run time).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     No entry point synchronises, except nvfp4lora_prepare (one documented device-to-
 *     host read) and nvfp4lora_device_status.
 *   - Arguments are checked on the host before anything is enqueued; a violation
 *     returns a status and enqueues nothing.  nvfp4lora_last_error() then names the
 *     violated rule.  No C++ exception crosses this boundary.
 *   - Only sm_100 (B200) is supported (mm_nvfp4_lora, Notes: Architectures).
 */
#ifndef NVFP4LORA_H
#define NVFP4LORA_H

#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4LORA_API __attribute__((visibility("default")))
#else
#define NVFP4LORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* nvfp4lora_stream;

typedef enum nvfp4lora_status {
    NVFP4LORA_OK = 0,
    /* Shape, pointer, alignment or size rule violated (mm_nvfp4_lora, Notes: Shape
     * rules): the Python layer turns it into ValueError, and the message names the rule. */
    NVFP4LORA_ERR_INVALID_ARG = 1,
    /* Prepared adapter used with another alpha, or its lora_b / lora_scale moved or
     * were written since the last (re)fold (mm_nvfp4_lora, Parameters: lora_adapter;
     * Notes: CUDA graphs -- StaleAdapterError). */
    NVFP4LORA_ERR_STALE_ADAPTER = 2,
    /* Eager prepare only: alpha == 0, or lora_scale / alpha is not finite
     * (prepare_nvfp4_lora_adapter, Parameters: alpha; Returns). */
    NVFP4LORA_ERR_ALPHA_ZERO = 3,
    /* The current device is not sm_100 (mm_nvfp4_lora, Notes: Architectures). */
    NVFP4LORA_ERR_UNSUPPORTED_ARCH = 4,
    /* A bounded wait inside a kernel ran out; reported by nvfp4lora_device_status. */
    NVFP4LORA_ERR_DEVICE_TIMEOUT = 5,
    /* A CUDA runtime / driver call failed; the message holds its error string. */
    NVFP4LORA_ERR_CUDA = 6
} nvfp4lora_status;

/*
 * A prepared (folded) adapter: prepare_nvfp4_lora_adapter's PreparedNvFp4LoraAdapter.
 * Plain data in host memory, owned by the caller.  b_folded and ratio are caller-owned
 * device buffers that the fold writes; the remaining fields are the "source pins"
 * checked by nvfp4lora_mm_prepared.
 */
typedef struct nvfp4lora_adapter {
    uint16_t*       b_folded;     /* bf16 [N, r] device: bf16_rne(lora_b * ratio)           */
    float*          ratio;        /* fp32 [1] device: div.rn(lora_scale, alpha[0]); 0 = zero adapter */
    const float*    alpha;        /* the alpha tensor the adapter was folded for (identity) */
    const uint16_t* lora_b;       /* source pins: pointers and version token at the last fold */
    const float*    lora_scale;
    int64_t         N;
    int64_t         r;
    uint64_t        src_version;  /* caller-defined token of the sources' contents          */
    int32_t         device;       /* CUDA device ordinal the adapter lives on               */
    int32_t         reserved;
} nvfp4lora_adapter;

/*
 * Raw path (mm_nvfp4_lora: opening formula; "Raw path" bullet; Parameters).
 *
 *   a       uint8 [M, K/2] row-major, two E2M1 codes per byte (low nibble first).
 *   b       uint8 [N, K/2] row-major (the product is a @ b^T).
 *   a_sf    UE4M3 scales of a, one per 16 K-elements, 128x4 swizzled, rows padded to a
 *           multiple of 128: a_sf_bytes >= ceil(M/128)*128*K/16 (larger is accepted).
 *   b_sf    the same for b: b_sf_bytes >= ceil(N/128)*128*K/16.
 *   alpha   fp32 [1]: alpha_base / (a_global_scale * b_global_scale).
 *   d       bf16 [M, r] row-major (LoRA-down output); lora_b bf16 [N, r] row-major.
 *   lora_scale  fp32 [1] or NULL.  NULL is the adapter-off call (d, lora_b, r are then
 *           ignored).  A device value equal to 0 takes the zero-adapter path: no LoRA
 *           work, output bitwise equal to the adapter-off call.
 *   bias    bf16 [N] or NULL; added in fp32 before the single rounding.
 *   out     bf16 [M, N] row-major, written once per element.
 * Rules: M >= 1, N >= 1, K >= 256 and K % 256 == 0; with an adapter, r % 8 == 0 and
 * 8 <= r <= 128; a, b, a_sf, b_sf, d, lora_b, out 16-byte aligned; alpha, lora_scale
 * 4-byte aligned; bias 2-byte aligned.
 * The fp32 combine is v = alpha*acc; v = fma(lora_scale, lora_acc, v); v += bias;
 * out = bf16_rne(v).  Graph-capturable (no host read, no allocation).
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_mm(
    const uint8_t* a, const uint8_t* b,
    const uint8_t* a_sf, int64_t a_sf_bytes,
    const uint8_t* b_sf, int64_t b_sf_bytes,
    const float* alpha,
    const uint16_t* d, const uint16_t* lora_b, const float* lora_scale, int64_t r,
    const uint16_t* bias, uint16_t* out,
    int64_t M, int64_t N, int64_t K,
    nvfp4lora_stream stream);

/*
 * Eager fold (prepare_nvfp4_lora_adapter with out=None: summary paragraph, Returns).
 * Reads lora_scale[0] and alpha[0] back to the host (the one documented host read; it
 * synchronises `stream`), refuses alpha == 0 or a non-finite ratio with
 * NVFP4LORA_ERR_ALPHA_ZERO, then enqueues the fold:
 *     ratio[0]    = div.rn.f32(lora_scale[0], alpha[0])
 *     b_folded[i] = bf16_rne(fp32(lora_b[i]) * ratio)       (NaN stored as 0x7FC0)
 * and fills *adapter_out (pins: alpha, lora_b, lora_scale, src_version, device).
 *   lora_b     bf16 [N, r] device, 16-byte aligned; r % 8 == 0, 8 <= r <= 128.
 *   b_folded   bf16 [N, r] device, caller-allocated, 16-byte aligned.
 *   ratio      fp32 [1] device, caller-allocated.
 * On error nothing is enqueued and *adapter_out is left unchanged.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_prepare(
    const uint16_t* lora_b, const float* lora_scale, const float* alpha,
    int64_t N, int64_t r,
    uint16_t* b_folded, float* ratio, uint64_t src_version,
    nvfp4lora_adapter* adapter_out,
    nvfp4lora_stream stream);

/*
 * In-place refold (prepare_nvfp4_lora_adapter with out=adapter; Parameters: out).
 * Same arithmetic as the eager form, bitwise, computed entirely on the device: no host
 * read, graph-capturable.  alpha must be adapter->alpha (else INVALID_ARG); lora_b must
 * keep the adapter's N, r and device; lora_scale may be a new tensor.  The pins are
 * refreshed to (lora_b, lora_scale, src_version).  alpha == 0 is not refused here: the
 * ratio is stored as IEEE division gives it and propagates into the GEMM.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_refold(
    nvfp4lora_adapter* adapter,
    const uint16_t* lora_b, const float* lora_scale, const float* alpha,
    int64_t N, int64_t r, uint64_t src_version,
    nvfp4lora_stream stream);

/*
 * Prepared path (mm_nvfp4_lora: "Prepared path" bullet; Parameters: lora_adapter).
 * Accumulates the base product, then d @ b_folded^T into the same fp32 accumulator,
 * and applies alpha once: v = alpha*acc; v += bias; out = bf16_rne(v).  A zero ratio
 * (lora_scale == 0 at the last fold) gives the adapter-off output bitwise.
 * Stale checks (NVFP4LORA_ERR_STALE_ADAPTER): alpha != adapter->alpha, or
 * cur_lora_b / cur_lora_scale / cur_src_version differ from the adapter's pins.
 * d is bf16 [M, adapter->r]; the other arguments are as for nvfp4lora_mm.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_mm_prepared(
    const uint8_t* a, const uint8_t* b,
    const uint8_t* a_sf, int64_t a_sf_bytes,
    const uint8_t* b_sf, int64_t b_sf_bytes,
    const float* alpha, const uint16_t* d,
    const nvfp4lora_adapter* adapter,
    const uint16_t* cur_lora_b, const float* cur_lora_scale, uint64_t cur_src_version,
    const uint16_t* bias, uint16_t* out,
    int64_t M, int64_t N, int64_t K,
    nvfp4lora_stream stream);

/*
 * Grouped (expert-partitioned) call: flashinfer.grouped_mm.grouped_mm_bf16's formula
 * (out[start:end] = a[start:end] x b[e]^T for each expert e, start, end = m_indptr[e],
 * m_indptr[e+1]) applied to the operation of nvfp4lora_mm, segment by segment:
 *     out[s:t] = bf16_rne( alpha[e] * (dequant(a[s:t]) @ dequant(b[e])^T)
 *                          + lora_scale * (d[s:t] @ lora_b[e]^T) [+ bias[e]] )
 *   a       uint8 [rows, K/2]; a_sf its UE4M3 scales in the 128x4 layout over all rows
 *           (a_sf_bytes >= ceil(rows/128)*128*K/16).
 *   b       uint8 [num_experts, N, K/2]; b_sf num_experts consecutive 128x4 buffers of N rows
 *           (b_sf_bytes >= num_experts*ceil(N/128)*128*K/16).
 *   m_indptr int32 [num_experts + 1] device, read on the device (no host read, graph-capturable).
 *           Reading taken (the pages define the grouped form for bf16 only): m_indptr[0] == 0, the
 *           entries are non-decreasing multiples of 128 and m_indptr[E] <= rows, so each expert's
 *           rows fill whole 128-row blocks of the scale layout; padding rows inside a segment are
 *           computed like any other row, rows from m_indptr[E] on are neither read nor written.
 *           A table that breaks these rules computes nothing and makes the next
 *           nvfp4lora_device_status return NVFP4LORA_ERR_INVALID_ARG.
 *   alpha   fp32 [num_experts] device (each expert's alpha_base / (a_gs * b_gs[e])).
 *   d       bf16 [rows, r]; lora_b bf16 [num_experts, N, r]; lora_scale fp32 [1] or NULL (adapter
 *           off; a device value of 0 does no LoRA work and gives the adapter-off output bitwise).
 *   bias    bf16 [num_experts, N] or NULL.   out bf16 [rows, N].
 * Rules as for nvfp4lora_mm (alignment, K % 256 == 0, r), 1 <= num_experts <= 511.  The raw
 * combine of nvfp4lora_mm applies per segment.  Enqueued on `stream`.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_grouped_mm(
    const uint8_t* a, const uint8_t* b,
    const uint8_t* a_sf, int64_t a_sf_bytes,
    const uint8_t* b_sf, int64_t b_sf_bytes,
    const int32_t* m_indptr, int64_t num_experts,
    const float* alpha,
    const uint16_t* d, const uint16_t* lora_b, const float* lora_scale, int64_t r,
    const uint16_t* bias, uint16_t* out,
    int64_t rows, int64_t N, int64_t K,
    nvfp4lora_stream stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error word that
 * kernels set when one of their bounded waits runs out (NVFP4LORA_ERR_DEVICE_TIMEOUT) or
 * when a table read on the device breaks its rules (a grouped call's m_indptr, a LoRA delta's
 * routing: NVFP4LORA_ERR_INVALID_ARG).  Returns NVFP4LORA_OK when the word was clear (or
 * NVFP4LORA_ERR_CUDA).
 * The GEMM, fold and quantize calls return NVFP4LORA_OK once their work is enqueued; a kernel
 * whose bounded wait gives up returns early and leaves its outputs (out, b_folded, ratio, codes,
 * scales) partly unwritten.  Their contents are therefore defined only once a later
 * nvfp4lora_device_status on the same stream has returned NVFP4LORA_OK.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_device_status(nvfp4lora_stream stream);

/*
 * Self-test of the failure path of the bounded waits (the pages have no counterpart; it lets a
 * test exercise the path without faulting the GPU).  Enqueues on `stream` one CTA that waits
 * on an mbarrier nothing completes, with the same wait helper as the GEMM kernels and a limit
 * of limit_ns nanoseconds (0 < limit_ns <= 1e9) instead of 2 s.  The wait runs out and raises
 * the device error word; the kernel then returns, so the context stays usable.  The next
 * nvfp4lora_device_status returns NVFP4LORA_ERR_DEVICE_TIMEOUT and clears the word.
 * Returns NVFP4LORA_ERR_INVALID_ARG (nothing enqueued) for a limit out of range.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_selftest_wait_timeout(int64_t limit_ns, nvfp4lora_stream stream);

/*
 * NVFP4 quantizer: the producer of a / a_sf that the mm_nvfp4_lora page names (the paragraph
 * after the formula: the operands come in the 128x4 swizzled layout that fp4_quantize writes;
 * Parameters: alpha = alpha_base / (a_global_scale * b_global_scale)).  The pages give no rule; this library
 * computes, per 16-element block along K, in float32:
 *     amax = max |x|;  sf = E4M3(rne, saturating at 448)((amax * gs) / 6);
 *     code = E2M1(rne, saturating at 6)(x * (gs / value(sf)))   (sf == 0: +0 codes),
 * so value(code) * value(sf) / gs approximates x.
 *   x       bf16 [rows, K] device, row-major, 16-byte aligned.  Finite values.
 *   global_scale  fp32 [1] device, 4-byte aligned: gs, positive and finite (read on the device;
 *           no host read).
 *   codes   uint8 [rows, K/2] device, caller-owned, 16-byte aligned: element 2j of a row in the
 *           low nibble of byte j.
 *   scales  uint8 device, caller-owned, 16-byte aligned, scales_bytes >= ceil(rows/128)*128*(K/16):
 *           the 128x4 swizzled layout; the bytes of padded rows are written as 0.
 * K % 64 == 0 (whole scale atoms).  Enqueued on `stream`; NVFP4LORA_ERR_INVALID_ARG (nothing
 * enqueued) for a rule violation.  The pages have no counterpart for the exact rule.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_quantize(
    const uint16_t* x, int64_t rows, int64_t K, const float* global_scale,
    uint8_t* codes, uint8_t* scales, int64_t scales_bytes,
    nvfp4lora_stream stream);

/* Element types of the routed-MoE LoRA delta's activation, banks and output. */
typedef enum nvfp4lora_dtype {
    NVFP4LORA_DTYPE_BF16 = 0,
    NVFP4LORA_DTYPE_FP16 = 1
} nvfp4lora_dtype;

/*
 * Routed-MoE FC2 (down projection) LoRA delta: flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta
 * (opening formula and Parameters).  For every token t with adapter l = lora_ids[t]:
 *     out[t] = scale * sum_j topk_weights[t, j] * ( B_down[l, e] @ ( A_down[l, e] @ act[p] ) )
 * over its routed slots j (e = topk_ids[t, j], p = expanded_idx_to_permuted_idx[t*top_k + j]),
 * to be added to the MoE output by the caller.  Readings taken where the page is silent:
 * A_down[l, e] is the [rank, I] row-major block that starts l*lora_stride_a elements after
 * w_ptr_a[e]; B_down[l, e] the [H, rank] row-major block l*lora_stride_b elements after
 * w_ptr_b[e]; act and both banks hold lora_dtype values; a negative lora id gives an all-zero
 * row; a negative permuted index is an inactive slot; the sum is formed in fp32 and rounded once
 * to out_dtype (nearest, ties to even).
 *   act      lora_dtype [padded_rows, I] device, row-major, 16-byte aligned (the permuted
 *            post-activation rows of the MoE's first GEMM).  I % 8 == 0.
 *   expanded_idx_to_permuted_idx  int32 [num_tokens * top_k] device.
 *   w_ptr_a, w_ptr_b  int64 [num_experts] device tables of bank addresses (device memory of
 *            this GPU, caller-owned and alive until the call completes); a bank address plus
 *            l * stride * 2 bytes must be 16-byte aligned, so lora_stride_a % 8 == 0 and
 *            lora_stride_b % 8 == 0.  Adapter ids must index adapters that exist in the banks:
 *            the library cannot see the banks' sizes.
 *   topk_ids int32 [num_tokens, top_k]; topk_weights fp32 [num_tokens, top_k];
 *   lora_ids int32 [num_tokens]; all device.
 *   rank     8 <= rank <= 128, rank % 8 == 0.   1 <= top_k <= 16.   hidden_size = H >= 1.
 *   out      out_dtype [num_tokens, H] device, caller-owned, fully written.
 * Every rule above that the host can see is checked before any CUDA call
 * (NVFP4LORA_ERR_INVALID_ARG, nothing enqueued).  Routing entries are read on the device: an
 * expert id outside [0, num_experts), a permuted index >= padded_rows or a bank address that
 * is null or misaligned is skipped, and the next nvfp4lora_device_status returns
 * NVFP4LORA_ERR_INVALID_ARG.  num_tokens == 0 enqueues nothing.  Enqueued on `stream`.
 */
NVFP4LORA_API nvfp4lora_status nvfp4lora_bgmv_moe_gemm2_lora_delta(
    const void* act, int64_t padded_rows, int64_t I,
    const int32_t* expanded_idx_to_permuted_idx,
    const int64_t* w_ptr_a, int64_t lora_stride_a,
    const int64_t* w_ptr_b, int64_t lora_stride_b,
    const int32_t* topk_ids, const float* topk_weights, const int32_t* lora_ids,
    int64_t num_tokens, int64_t top_k, int64_t num_experts,
    int64_t rank, int64_t hidden_size,
    int32_t lora_dtype, float scale, int32_t out_dtype,
    void* out, nvfp4lora_stream stream);

/* Message of the last failing call on this host thread ("" when none). */
NVFP4LORA_API const char* nvfp4lora_last_error(void);

/* Library version string. */
NVFP4LORA_API const char* nvfp4lora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4LORA_H */
