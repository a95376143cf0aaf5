/*
 * libsplitkv_attn — split-KV (replicated prefix + suffix), tail-padded,
 * non-causal bf16 attention for B200 (sm_100a), behind a plain C ABI.
 *
 * The operation (per batch row b, query head hq, query row i):
 *
 *   K* = cat(k_prefix[b, :, hkv], k_suffix[b, :, hkv])[0 : real_len[b]]
 *   V* = cat(v_prefix[b, :, hkv], v_suffix[b, :, hkv])[0 : real_len[b]]
 *   out[b, i, hq, :] = softmax(softmax_scale * q[b, i, hq, :] . K*^T) . V*
 *
 * with hkv = hq / (num_q_heads / num_kv_heads).  Sources:
 *  - "sglang PR 26973" (Cosmos3), layer.py, forward_with_replicated_kv_prefix:
 *    the K/V prefix (replicated across sequence-parallel ranks, e.g. text
 *    tokens) and suffix (e.g. video tokens) arrive as separate tensors and the
 *    result is attention over their concatenation along the sequence axis,
 *    prefix first.  This library never materialises that concatenation.
 *  - "sglang PR 30107" (unified SP shard utils), sp_shard_utils.py: padding is
 *    one contiguous block at the global sequence tail; tail_attn_meta's
 *    valid_len gives the number of real tokens (here: real_len[b]).  Pad keys
 *    are excluded from the softmax and are never read.
 *  - "vLLM-Omni performance patterns", shared Attention wiring: BSND layout,
 *    GQA (num_heads % num_kv_heads == 0), softmax_scale = head_dim ** -0.5 as
 *    the usual value, causal = False.
 *  - "sglang PR 26973", cosmos3video.py: q/k/v may be strided views of one
 *    fused projection output [B, S, Hq + 2*Hkv, D] (view + slice, no copy).
 *
 * Conventions for every entry point:
 *  - Tensors are bf16, layout BSND, described by sk_tensor_t; the head_dim
 *    axis is contiguous (stride 1).  All strides are in elements.
 *  - Device pointers are owned by the caller; the library keeps no reference
 *    after the call returns and allocates no device memory.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without synchronising.  A call made while
 *    the stream is being captured into a CUDA graph is captured.
 *  - Host arrays (real_len, q_valid) are read before the call returns.
 *  - A non-OK status means nothing was launched (except SK_ERR_CUDA from a
 *    failed launch); sk_last_error() then returns a message for this thread.
 *  - No C++ exception crosses this interface.
 */
#ifndef SPLITKV_ATTN_H
#define SPLITKV_ATTN_H

#include <stdint.h>

#if defined(__GNUC__)
#define SK_API __attribute__((visibility("default")))
#else
#define SK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SK_OK = 0,
  SK_ERR_INVALID_ARG = 1,    /* bad sizes, strides, alignment, ranges, aliasing */
  SK_ERR_UNSUPPORTED = 2,    /* valid request the library does not serve (head_dim, device) */
  SK_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed */
  SK_ERR_DEVICE_TIMEOUT = 4  /* a kernel gave up a bounded wait (see sk_device_status) */
} sk_status_t;

/* One BSND bf16 tensor (or strided view).  Element (b, s, h, d) lives at
 * ptr + b*stride_b + s*stride_s + h*stride_h + d.  ptr must be 16-byte
 * aligned and stride_b, stride_s, stride_h multiples of 8 elements (16 bytes,
 * the TMA rule).  The head count comes from the call's num_*_heads. */
typedef struct {
  void* ptr;        /* device address of element (0,0,0,0); may be NULL when len_s == 0 */
  int64_t stride_b; /* elements between batch rows */
  int64_t stride_s; /* elements between sequence positions */
  int64_t stride_h; /* elements between heads */
  int32_t len_s;    /* sequence length of this tensor */
} sk_tensor_t;

/*
 * attn_fwd_split_kv — forward attention over cat(prefix, suffix) clipped to
 * real_len, without the concatenation.
 *
 *   q         [batch, Sq, num_q_heads, head_dim]        (read)
 *   k_prefix, v_prefix [batch, Sp, num_kv_heads, head_dim] (read; Sp may be 0)
 *   k_suffix, v_suffix [batch, Ss, num_kv_heads, head_dim] (read; Ss may be 0)
 *   real_len  HOST int32[batch]: valid keys of row b counted in prefix-then-
 *             suffix order, 0 <= real_len[b] <= Sp + Ss.  NULL = all Sp + Ss.
 *             Keys j >= real_len[b] may hold any bits (NaN, Inf): they are
 *             never loaded.
 *   softmax_scale  finite, >= 0 (usually head_dim ** -0.5).
 *   out       [batch, Sq, num_q_heads, head_dim] (written); must not overlap
 *             any input or itself.
 *   head_dim  64 or 128.
 *
 * Query rows: when Sq == Sp + Ss (joint self-attention, where queries and
 * keys are the same padded token stream) rows i >= real_len[b] are pad;
 * otherwise every row is real.  Pad rows and rows of a batch row with no
 * valid key are written as exact zeros; no other bytes of `out` are written.
 * The normaliser is fp32; the output is rounded to bf16 (nearest even).
 * Returns SK_OK, SK_ERR_INVALID_ARG, SK_ERR_UNSUPPORTED or SK_ERR_CUDA.
 */
SK_API sk_status_t attn_fwd_split_kv(const sk_tensor_t* q, const sk_tensor_t* k_prefix,
                              const sk_tensor_t* v_prefix, const sk_tensor_t* k_suffix,
                              const sk_tensor_t* v_suffix, const int32_t* real_len,
                              int32_t num_q_heads, int32_t num_kv_heads, float softmax_scale,
                              const sk_tensor_t* out, int32_t batch, int32_t head_dim,
                              void* stream);

/*
 * attn_fwd_split_kv_ex — as attn_fwd_split_kv, with an explicit HOST
 * int32[batch] q_valid (0 <= q_valid[b] <= Sq): rows i >= q_valid[b] are pad
 * and written as zeros.  q_valid == NULL applies the rule above.
 */
SK_API sk_status_t attn_fwd_split_kv_ex(const sk_tensor_t* q, const sk_tensor_t* k_prefix,
                                 const sk_tensor_t* v_prefix, const sk_tensor_t* k_suffix,
                                 const sk_tensor_t* v_suffix, const int32_t* real_len,
                                 int32_t num_q_heads, int32_t num_kv_heads, float softmax_scale,
                                 const sk_tensor_t* out, int32_t batch, int32_t head_dim,
                                 const int32_t* q_valid, void* stream);

/*
 * attn_fwd_split_kv_scatter — as attn_fwd_split_kv_ex, with the output
 * all-to-all of the Ulysses form fused into the store ("sglang PR 26973",
 * _forward_with_replicated_kv_prefix_split: head-sharded attention, then an
 * all-to-all of the output from head shards back to sequence shards).  The
 * query stream is the gathered sequence of num_dst equal chunks; output row s
 * of batch row b and (local) query head h is written to
 *
 *   dst[s / L] + b*dst_layout.stride_b + (s % L)*dst_layout.stride_s
 *              + (head_offset + h)*dst_layout.stride_h,   L = dst_layout.len_s
 *
 * i.e. straight into the receive buffer of the rank that owns that chunk, at
 * this rank's head slot.  Each tile's rows are stored as soon as the tile is
 * done, so the exchange overlaps the attention of later tiles.
 *
 *   dst        HOST array of num_dst (1..8) device addresses, 16-byte aligned.
 *              They may be other GPUs' memory mapped into this process (CUDA
 *              IPC, symmetric memory); the kernel issues only plain stores to
 *              them, all performed by the time it completes in stream order.
 *              The caller owns the buffers and orders the readers after that
 *              point: a barrier across ranks enqueued on `stream` after this
 *              call (an NCCL collective signals its peers only after the work
 *              before it on the stream has completed).
 *   dst_layout strides of every destination (ptr ignored); len_s = L >= 1,
 *              and num_dst * L must equal q.len_s.  Heads head_offset ..
 *              head_offset + num_q_heads - 1 of each destination are written
 *              (pad rows as zeros); nothing else is touched.
 * Destinations are not checked for overlap with the inputs (they may live on
 * other devices); the caller keeps them apart.  Other arguments and errors as
 * attn_fwd_split_kv_ex.
 */
SK_API sk_status_t attn_fwd_split_kv_scatter(const sk_tensor_t* q, const sk_tensor_t* k_prefix,
                                      const sk_tensor_t* v_prefix, const sk_tensor_t* k_suffix,
                                      const sk_tensor_t* v_suffix, const int32_t* real_len,
                                      const int32_t* q_valid, int32_t num_q_heads, int32_t num_kv_heads,
                                      float softmax_scale, void* const* dst, int32_t num_dst,
                                      const sk_tensor_t* dst_layout, int32_t head_offset, int32_t batch,
                                      int32_t head_dim, void* stream);

/*
 * attn_fwd_varlen — packed variable-length attention: several independent
 * sequences (segments) concatenated along one token axis, each attending only
 * to its own keys (a block-diagonal mask, never materialised).  Sources:
 * "vLLM-Omni performance patterns" (packed varlen attention driven by
 * cu_seqlens computed once on the host, validated against dense attention
 * with unequal sample lengths and padding exclusion) and "sglang PR 30107"
 * (varlen FlashAttention over [valid | pad] segments).
 *
 *   q    [1, Tq, num_q_heads, head_dim]  (read; stride_b ignored)
 *   k, v [1, Tk, num_kv_heads, head_dim] (read)
 *   cu_seqlens_q, cu_seqlens_k  HOST int32[num_segments + 1], non-decreasing,
 *        cu[0] >= 0, cu_q[n] <= Tq, cu_k[n] <= Tk.  Segment i owns query rows
 *        [cu_q[i], cu_q[i+1]) and key rows [cu_k[i], cu_k[i+1]).
 *   seqused_q, seqused_k  HOST int32[num_segments] or NULL: the first
 *        seqused_*[i] rows of segment i are valid (the rest is pad: pad keys
 *        are never loaded, pad query rows are written as zeros).  NULL = all.
 *   softmax_scale  finite, >= 0.   head_dim  64 or 128.
 *   out  [1, Tq, num_q_heads, head_dim] (written on the segments' rows only;
 *        rows outside every segment are not touched); must not overlap the
 *        inputs or itself.
 * A segment with no valid key writes zeros.  One kernel launch per 1024
 * segments (the segments of a launch are processed longest first), on
 * `stream`.  Returns SK_OK, SK_ERR_INVALID_ARG, SK_ERR_UNSUPPORTED or
 * SK_ERR_CUDA.
 */
SK_API sk_status_t attn_fwd_varlen(const sk_tensor_t* q, const sk_tensor_t* k, const sk_tensor_t* v,
                                   const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                   const int32_t* seqused_q, const int32_t* seqused_k,
                                   int32_t num_segments, int32_t num_q_heads, int32_t num_kv_heads,
                                   float softmax_scale, const sk_tensor_t* out, int32_t head_dim,
                                   void* stream);

/*
 * qk_rmsnorm_rope — fused Q/K RMSNorm over head_dim followed by rotary
 * embedding, in place on q and k (which may be strided views of one fused
 * QKV buffer).  Source: "vLLM-Omni performance patterns", Q/K RMSNorm + RoPE
 * (fused_qk_norm_rope with a non-interleaved [cos | sin] table; is_neox_style
 * False means interleaved pairs; partial rotary passes the rest through;
 * bf16 rounding where the unfused path stores bf16), and "sglang PR 26973",
 * cosmos3video.py (F.rms_norm with the norm weight and epsilon, then RoPE).
 *
 * For every token (b, s) and head of q (num_q_heads) and k (num_kv_heads):
 *   y_d = bf16(x_d / sqrt(mean(x^2) + eps) * w_d)          (w = w_q or w_k)
 *   pairs (a, c) = (i, i + rot_dim/2) when interleaved == 0, (2i, 2i+1) otherwise,
 *   i < rot_dim/2, with cs = rope_table[s, i], sn = rope_table[s, rot_dim/2 + i]:
 *     x_a <- bf16(y_a*cs - y_c*sn),  x_c <- bf16(y_c*cs + y_a*sn)
 *   dims d >= rot_dim: x_d <- y_d.
 *   q, k       [batch, S, heads, head_dim] bf16 (read and written in place)
 *   w_q, w_k   device bf16[head_dim]
 *   rope_table device fp32[table_rows, rot_dim] ([cos | sin]), table_rows >= S
 *   rot_dim    even, 0 <= rot_dim <= head_dim;  head_dim in {64, 128, 256}
 *   eps        >= 0
 *   exact      0: evaluate the formula above in fp32 (sum of squares and
 *              1/sqrt in fp32, both bf16 rounding points kept), bound by
 *              memory bandwidth; each rotated result lies within three bf16
 *              ulps, taken at the magnitude of its own two terms (|y_a*cs| +
 *              |y_c*sn| for x_a, |y_c*cs| + |y_a*sn| for x_c), of the same
 *              formula evaluated exactly with those two roundings (two for a
 *              rare one-ulp difference in y carried through, one for the
 *              final roundings); dims past rot_dim within one ulp of y.
 *              1: return exactly the bits of that exact evaluation (fp32 with
 *              an error bound, elements the bound cannot decide redone in
 *              fp64), about twice as slow.
 * Returns SK_OK, SK_ERR_INVALID_ARG, SK_ERR_UNSUPPORTED or SK_ERR_CUDA.
 */
SK_API sk_status_t qk_rmsnorm_rope(const sk_tensor_t* q, const sk_tensor_t* k, const void* w_q,
                            const void* w_k, const float* rope_table, int32_t table_rows,
                            int32_t rot_dim, int32_t interleaved, float eps,
                            int32_t num_q_heads, int32_t num_kv_heads, int32_t batch,
                            int32_t head_dim, int32_t exact, void* stream);

/*
 * sk_shard_pad_copy — one rank's chunk of a tail-padded sequence shard
 * ("sglang PR 30107", shard_like: pad the tail of the stream with num_pad rows
 * of zeros or repeats of its last row, then take rows [first_row,
 * first_row + dst_rows)), in one pass that reads only the chunk's real rows.
 * Needed only on the rank whose chunk holds pad; other chunks are views.
 *
 *   src   device, rows of row_bytes bytes: row s of batch b at
 *         src + b*src_stride_b + s*src_stride_s, s < src_rows (read)
 *   dst   device, dst_rows rows per batch row at dst + b*dst_stride_b +
 *         r*dst_stride_s (written); must not overlap src or itself
 *   row   r of dst = src row first_row + r if < src_rows, else zeros
 *         (pad_mode 0) or src row src_rows - 1 (pad_mode 1)
 *   row_bytes and all strides multiples of 16, pointers 16-byte aligned.
 * Returns SK_OK, SK_ERR_INVALID_ARG or SK_ERR_CUDA; launches on `stream`.
 */
SK_API sk_status_t sk_shard_pad_copy(const void* src, int64_t src_stride_b, int64_t src_stride_s,
                                     int32_t src_rows, void* dst, int64_t dst_stride_b,
                                     int64_t dst_stride_s, int32_t dst_rows, int32_t first_row,
                                     int32_t row_bytes, int32_t batch, int32_t pad_mode, void* stream);

/* Message for the last non-OK status returned on this host thread ("" if none). */
SK_API const char* sk_last_error(void);

/*
 * sk_device_status — synchronises `device` and reads the library's device
 * status word: 0, or SK_ERR_DEVICE_TIMEOUT if any kernel since the last clear
 * gave up a bounded wait (its outputs are then undefined; the context stays
 * usable).  clear != 0 resets the word.  Returns SK_OK or SK_ERR_CUDA.
 */
SK_API sk_status_t sk_device_status(int32_t device, int32_t* status_out, int32_t clear);

/* Bound on every in-kernel wait, in milliseconds (default 2000; 1..60000). */
SK_API sk_status_t sk_set_wait_timeout_ms(int32_t ms);

/*
 * sk_test_stall_mma — test hook for the failure path (no counterpart on the
 * pages).  While on != 0, the attention kernels' MMA warp first waits on a
 * barrier that nothing arrives at, so every in-kernel wait runs out after the
 * sk_set_wait_timeout_ms limit: each CTA raises SK_ERR_DEVICE_TIMEOUT in the
 * device status word, drains its own copies, frees TMEM and exits, and the
 * context stays usable.  Outputs of such calls are undefined.  Off by default;
 * returns SK_OK.
 */
SK_API sk_status_t sk_test_stall_mma(int32_t on);

/* ABI version of this header (increments on incompatible change). */
SK_API int32_t sk_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPLITKV_ATTN_H */
