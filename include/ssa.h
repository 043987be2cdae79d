/*
 * ssa.h -- C ABI of libssa: the skip-softmax / N:M sparse flash-attention
 * forward pass on NVIDIA B200 (sm_100a).
 *
 * The method (cited by page title and section):
 *   - "Skip-Softmax Sparse Attention for Diffusion Models" (Model-Optimizer
 *     examples/diffusers/sparsity README), intro: skip-softmax (BLASST) skips
 *     KV tiles whose attention scores are negligible during the FlashAttention
 *     computation; "Threshold Modes" table: the kernel receives the lambda
 *     threshold and compares in the log2 domain (log2(lambda)).  A (Br x Bc)
 *     tile is skipped when exp(tile_row_max - running_max) < lambda holds for
 *     every query row of the tile; a skipped tile issues no exp, no V load and
 *     no P.V product, and leaves the running max, sum and output untouched.
 *   - "Attention Sparsity for HuggingFace Models" (Model-Optimizer
 *     examples/llm_sparsity/attention_sparsity README), "N:M Sparse Softmax"
 *     and "Custom N:M configuration": for every M consecutive key positions
 *     keep the top-N scores and set the rest to -inf before softmax
 *     (M = 4 with N = 1..3, M = 8 with N = 1..7); the first
 *     dense_sink_tokens keys and a local window of dense_recent_tokens keys
 *     are kept dense; tile shape knobs br / bc.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     contiguous, owned by the caller; bf16 and fp32 tensors 16-byte aligned,
 *     int32 / uint32 arrays 4-byte aligned (SSA_ERR_INVALID_ARG otherwise).
 *     The library keeps no reference to them after the call returns.
 *   - q:   [B, Lq, Hq, d]  bf16
 *     k,v: [B, Lk, Hkv, d] bf16
 *     out: [B, Lq, Hq, d]  bf16 (overwritten)
 *     lse: [B, Hq, Lq]     fp32, natural-log log-sum-exp of the scaled scores
 *                          of the kept keys (-inf for a row with none)
 *     tile_skip_count: [B, Hq, nQ] int32, nQ = ceil(Lq / Br): number of
 *                          visited key tiles skipped by each query tile
 *                          (overwritten, not accumulated).
 *   - Query head hq reads KV head hq / (Hq / Hkv) (grouped-query attention).
 *   - causal != 0: bottom-right aligned mask, query row i sees keys
 *     j <= i + (Lk - Lq).  Key tiles wholly above the diagonal are never
 *     visited and are not counted.
 *   - scores are scale * q.k; scale > 0 and finite.
 *   - mode: bit 0 (SSA_MODE_SKIP) enables the tile skip with threshold
 *     lambda (>= 0; 0 never skips); bit 1 (SSA_MODE_NM) enables N:M with
 *     n, m, sink, recent.  Parameters of a disabled mode are ignored.
 *     N:M groups are aligned to key 0; the recent window of row i is the keys
 *     0 <= pos_i - j < recent.  n == m is accepted (it keeps every key).
 *   - Br, Bc in {64, 128}; d in {64, 128}.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Argument errors are reported synchronously,
 *     before anything is launched; no exception crosses this boundary.
 *   - A device-side wait that times out (it never should) makes the kernel
 *     unwind and record SSA_ERR_TIMEOUT in a per-device status word, read by
 *     ssa_device_status().
 */
#ifndef SSA_H
#define SSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSA_OK 0
#define SSA_ERR_INVALID_ARG (-1) /* null pointer, non-positive size, bad lambda/scale, misalignment */
#define SSA_ERR_UNSUPPORTED (-2) /* d, Br, Bc, n/m outside the supported set */
#define SSA_ERR_CUDA (-3)        /* a CUDA runtime/driver call failed (launch, tensor map) */
#define SSA_ERR_TIMEOUT (-4)     /* a device-side bounded wait expired */

#define SSA_MODE_DENSE 0
#define SSA_MODE_SKIP 1
#define SSA_MODE_NM 2

/* Forward pass.  Returns SSA_OK once the kernel is enqueued, or a negative
 * status (nothing enqueued) for invalid or unsupported arguments. */
int ssa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
            int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
            float scale, int mode, float lambda, int n, int m, int sink, int recent, int Br, int Bc,
            void* stream);

/* Same kernel as ssa_fwd, also writing per-tile evidence (any may be NULL):
 *   skip_bits: [B, Hq, nQ, ceil(nK / 32)] uint32, nK = ceil(Lk / Bc); bit kt of
 *              query tile qt is set iff key tile kt was visited and skipped.
 *              Every word of every query tile is written.
 *   keep_bits: [B, Hq, Lq, ceil(Lk / 32)] uint32; bit j of row i is set iff key
 *              j is visible to row i and kept by N:M (every visible key when N:M
 *              is off), for the key tiles the row's query tile visits.  Words of
 *              tiles that are not visited are not written: zero the buffer first.
 *   v_tile_loads: [B, Hq, ceil(nQp / 2)] int32, nQp = ceil(Lq / 128): the
 *              number of V tiles the CTA that owns query rows
 *              [256 p, 256 p + 256) of (b, hq) loaded.  The kernel loads V
 *              tile kt only once one of those rows' query tiles has decided to
 *              keep key tile kt, so this equals the number of key tiles kept by
 *              at least one of them (the evidence that a skipped tile never
 *              issues its V load).
 * Skipped tiles still report their keep bits (the N:M mask precedes the skip). */
int ssa_fwd_debug(const void* q, const void* k, const void* v, void* out, float* lse,
                  int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                  int causal, float scale, int mode, float lambda, int n, int m, int sink,
                  int recent, int Br, int Bc, void* stream, uint32_t* skip_bits,
                  uint32_t* keep_bits, int32_t* v_tile_loads);

/* Allocation-free variant of ssa_fwd (the pages have no counterpart; this is
 * a service of this library).  Same arguments, layouts and results as
 * ssa_fwd, and it never allocates device memory: no cudaMalloc, no cudaFree,
 * no allocating library routine.  It is meant for callers that cannot
 * allocate while they run -- an inference engine's plugin that must work
 * inside the memory it was given at build time, a process whose device memory
 * is wholly owned by a framework's pooling allocator, or a latency-critical
 * path that cannot afford the implicit device synchronisation of cudaMalloc.
 * ssa_fwd, by contrast, allocates a status word on its first call per device.
 *
 * Scratch: the kernel's status word (raised when a bounded device wait times
 * out) lives in a static 256-byte device array inside libssa, held by every
 * GPU that loads the library until the process exits.  One call needs 4
 * bytes of it whatever the problem size; a call needing more than 256 bytes
 * would be rejected with SSA_ERR_UNSUPPORTED.  The array is shared by every
 * call on a device and keeps the last call's contents: each call clears the
 * status word on `stream` before its kernel starts.  Calls that overlap on the
 * GPU (on different streams) therefore race on that word; serialise them.
 * A timed-out wait makes the kernel unwind and raise that word;
 * ssa_device_status (which allocates nothing either) reads and clears it.
 * The first call on a device looks up the array's device address (with that
 * device current); later calls reuse it.
 * Returns SSA_OK once enqueued, or the status codes of ssa_fwd. */
int ssa_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                    int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                    int causal, float scale, int mode, float lambda, int n, int m, int sink,
                    int recent, int Br, int Bc, void* stream);

/* Forward pass over caller-selected key blocks.  The block-sparse page of the
 * same stack ("Bitmask format": packed UInt32 exact-block bitmaps owned per
 * (batch, KV head, Q block), one bit per KV block, padding bits in the final
 * word ignored) gives the selection format; this entry consumes it on the
 * skip-softmax path.  Everything else is ssa_fwd's: modes, layouts, outputs.
 *   block_mask: [B, Hkv, nQ, ceil(nK / 32)] uint32, device, 4-byte aligned,
 *               nQ = ceil(Lq / Br), nK = ceil(Lk / Bc); bit kt of word kt / 32
 *               of (b, hkv, qt) selects key tile kt for query tile qt of every
 *               query head that reads KV head hkv.  Bits of key tiles the query
 *               tile cannot see (causal) and padding bits are ignored.
 * A key tile whose bit is clear is not visited: no scores, no exponentials, no
 * P.V, not counted in tile_skip_count; the skip-softmax recurrence (when
 * SSA_MODE_SKIP is set) runs over the selected tiles in ascending order.  A
 * query row with no selected visible key gets out = 0 and lse = -inf.
 * Omitted blocks are dropped, not approximated (no proxy compensation).
 * Limit: nK <= 2048 (SSA_ERR_UNSUPPORTED beyond).  Returns the status codes of
 * ssa_fwd; SSA_ERR_INVALID_ARG for a NULL or misaligned block_mask. */
int ssa_fwd_blockmask(const void* q, const void* k, const void* v, void* out, float* lse,
                      int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                      int causal, float scale, int mode, float lambda, int n, int m, int sink,
                      int recent, int Br, int Bc, const uint32_t* block_mask, void* stream);

/* Same kernel as ssa_fwd_blockmask, also writing evidence (either may be NULL):
 *   skip_bits:    [B, Hq, nQ, ceil(nK / 32)] uint32; bit kt of query tile qt is
 *                 set iff key tile kt was selected, visible, and skipped.  Bits
 *                 are OR-ed in: zero the buffer first.
 *   v_tile_loads: as in ssa_fwd_debug (V tiles loaded per CTA). */
int ssa_fwd_blockmask_debug(const void* q, const void* k, const void* v, void* out, float* lse,
                            int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                            int causal, float scale, int mode, float lambda, int n, int m, int sink,
                            int recent, int Br, int Bc, const uint32_t* block_mask, void* stream,
                            uint32_t* skip_bits, int32_t* v_tile_loads);

/* Forward pass over caller-selected key blocks with proxy compensation of the
 * omitted ones.  The PrimTS pull request page ("proxy compensation", "Bitmask
 * format") keeps the selected blocks exact and stands in for every omitted
 * KV block with two summaries the caller provides, the arithmetic mean of its
 * keys and the sum of its values, correcting the softmax denominator by the
 * number of tokens a summary represents (the true length of a final partial
 * block included); a block computed exactly is not counted again.  The page
 * gives no formula; this library reads it as: for query row i and an omitted
 * block b of n_b keys, s_ib = scale * q_i . kmean_b adds n_b * exp(s_ib) to
 * the denominator and exp(s_ib) * vsum_b to the numerator, as if each of its
 * n_b keys had the mean key.  lse is the log of that denominator.
 *   block_mask: as in ssa_fwd_blockmask (selects the exact blocks).
 *   kmean, vsum: [B, nK, Hkv, d] bf16, 16-byte aligned, nK = ceil(Lk / Bc): per
 *                key block (of Bc keys, the last one possibly shorter) the mean
 *                of its keys and the sum of its values.
 * Non-causal only, no skip-softmax and no N:M (SSA_ERR_UNSUPPORTED is not
 * reachable: there is no causal or mode argument).  Other layouts, limits and
 * status codes are those of ssa_fwd_blockmask; no skip counts are written. */
int ssa_fwd_blockmask_proxy(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                            int Hq, int Hkv, int Lq, int Lk, int d, float scale, int Br, int Bc,
                            const uint32_t* block_mask, const void* kmean, const void* vsum,
                            void* stream);

/* Total key tiles visited by all query tiles of one (batch, head) pair: a pure
 * function of the shape, used to turn skip counts into skip fractions and
 * executed FLOPs.  Returns -1 for invalid sizes. */
int64_t ssa_visited_tiles(int causal, int Lq, int Lk, int Br, int Bc);

/* Test and diagnosis knob: the limit, in nanoseconds, of each pipeline wait
 * inside the kernel (an mbarrier wait for a TMA load, an MMA result, a
 * softmax hand-off).  0 restores the default (2 s).  When a wait gives up the
 * CTA unwinds: it records SSA_ERR_TIMEOUT, waits (with a separate, fixed 2 s
 * limit) for its own TMA loads and MMAs to finish, frees its tensor memory
 * and exits, so the context stays usable.  A tiny limit forces that path
 * without any fault; its outputs are then undefined.  Process-wide; takes
 * effect at the next launch. */
void ssa_set_wait_timeout_ns(uint64_t ns);

/* Synchronises `stream`, returns SSA_OK or SSA_ERR_TIMEOUT if a kernel on this
 * device recorded a timed-out wait since the last call (in the status word of
 * the allocating entry points or in that of ssa_fwd_noalloc), and clears the
 * word.  Allocates nothing.  Returns SSA_ERR_CUDA if the synchronisation
 * itself fails. */
int ssa_device_status(void* stream);

/* Decode-phase skip-softmax attention: a few query rows per sequence (Lq,
 * e.g. 1 new token, or a handful of speculative ones) against a long KV cache.
 * "Attention Sparsity for HuggingFace Models" (custom configuration) gives
 * skip-softmax separate prefill and decode thresholds; N:M is prefill only,
 * so there is no N:M here.  Layouts, GQA mapping, the bottom-right causal
 * mask, scale and lambda are those of ssa_fwd; the query tile is the Lq rows
 * of one query head (Lq <= Br), so a key tile is skipped for a head when
 * exp(tile_row_max - running_max) < lambda for each of its rows.
 *
 * The key tiles of each sequence are split into num_splits contiguous ranges
 * of ceil(nK / num_splits) tiles, nK = ceil(Lk / Bc), processed in parallel.
 * Each range runs the skip-softmax recurrence with its OWN running max (its
 * first tile is never skipped unless fully masked), and the ranges are merged
 * by the log-sum-exp rule.  With num_splits == 1 this is exactly ssa_fwd's
 * rule for one query tile; with more splits it is this reading of the method
 * for split-KV decoding (the pages do not define one), and skip decisions can
 * differ from the single-range ones.
 *
 *   tile_skip_count: [B, Hq] int32, skipped key tiles per (batch, head),
 *                    summed over splits (overwritten).
 *   workspace:       device scratch of at least ssa_decode_workspace_bytes()
 *                    bytes, 16-byte aligned, owned by the caller; holds the
 *                    partial results between the two kernels (four per
 *                    split and query row: accumulator, max and sum).
 *   Limits: d in {64, 128}, Bc in {64, 128}, (Hq / Hkv) * Lq <= 32
 *   (SSA_ERR_UNSUPPORTED otherwise); num_splits >= 1 (splits past the last
 *   key tile are empty and harmless).
 * Two kernels are enqueued on `stream`; no device memory is allocated.
 * Returns SSA_OK once enqueued, SSA_ERR_INVALID_ARG / SSA_ERR_UNSUPPORTED
 * (nothing enqueued) or SSA_ERR_CUDA. */
int ssa_decode(const void* q, const void* k, const void* v, void* out, float* lse,
               int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
               float scale, float lambda, int Bc, int num_splits, void* workspace,
               size_t workspace_bytes, void* stream);

/* Same kernels as ssa_decode, also writing the skip decisions:
 *   skip_bits: [B, Hq, ceil(nK / 32)] uint32 (non-NULL); bit kt of (b, hq) is
 *              set iff key tile kt was skipped for query head hq (by the split
 *              that owns it).  Bits are OR-ed in: zero the buffer first. */
int ssa_decode_debug(const void* q, const void* k, const void* v, void* out, float* lse,
                     int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
                     float scale, float lambda, int Bc, int num_splits, void* workspace,
                     size_t workspace_bytes, void* stream, uint32_t* skip_bits);

/* Bytes of workspace ssa_decode needs for this shape (0 for invalid sizes). */
size_t ssa_decode_workspace_bytes(int B, int Hq, int Lq, int d, int num_splits);

/* A num_splits for ssa_decode on a GPU with num_sms SMs.  The decode kernel is
 * persistent: one CTA per SM takes the B * Hkv * num_splits work items
 * (split, KV head, sequence) round-robin.  Returned: the split count s, at
 * most 256 and at most nK = ceil(Lk / Bc), that minimises the work of the
 * busiest CTA, ceil(B * Hkv * s / num_sms) * (ceil(nK / s) + 1) key tiles
 * (one tile's worth per split for its query rows, partial results and
 * merge); counts that would leave a split empty are passed over and ties go
 * to fewer splits.  Host only.  0 for invalid arguments (Bc not 64 or 128,
 * or a non-positive size). */
int ssa_decode_default_splits(int B, int Hkv, int Lk, int Bc, int num_sms);

/* Human-readable name of a status code (static storage). */
const char* ssa_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int ssa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H */
