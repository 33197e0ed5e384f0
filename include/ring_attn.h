/*
 * ring_attn.h -- C ABI of the B200 (sm_100a) ring-ordered blockwise attention
 * library (libring_attn.so).
 *
 * The operation follows "Ring Attention 环注意力" (slowleelab, ai-terms-fun):
 * the sequence of length L is cut into n_ring equal blocks (L4 §4.2 setup);
 * the query block of host i visits the K/V blocks in ring order
 * (i - t) mod n_ring for t = 0..n_ring-1 (L3 definition, L4 §4.2); every
 * visit is exact blockwise attention whose partial result is folded into a
 * running online-softmax accumulator (L4 §4.3), and under causal masking the
 * later blocks are skipped (L4 §4.5, limitation 2).  ring_attn_fwd and
 * ring_attn_bwd emulate the n_ring hosts as n_ring sequence blocks on one GPU;
 * ring_attn_fwd_visit and ring_attn_bwd_visit are one host's step of a ring
 * spread over devices, whose exchange the caller performs.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never frees or retains them after the call returns.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream).  Argument errors are reported synchronously, before anything is
 *     launched; device-side failures are reported by ring_attn_check_status.
 *   - No C++ exception crosses the ABI.  A non-OK status leaves a one-line
 *     explanation that ring_attn_last_error() returns (per host thread).
 *   - The library holds no device allocation of its own except static
 *     device variables of the module: three status words per device (bf16
 *     forward, backward and FP8 forward kernels), the fixed 4 MiB array of
 *     ring_attn_bwd_noalloc, and 64 work-queue counters.  Each kernel launch
 *     (one per forward call, two per backward call) takes the next counter
 *     in rotation and zeroes it with a memset ordered on `stream`, so up to
 *     64 launches may be in flight on different streams at once, and CUDA
 *     graph replays start from zero.
 *   - Contexts: a call runs in the calling thread's current CUDA context,
 *     the device's primary context or one the caller created (cuCtxCreate),
 *     and `stream` must belong to that context.  A thread with no current
 *     context gets the primary context of its current device made current.
 */
#ifndef RING_ATTN_H_
#define RING_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t / CUstream. */
typedef struct CUstream_st* ra_stream_t;

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID_ARG = 1,  /* a shape, pointer, alignment or value is invalid   */
  RA_ERR_UNSUPPORTED = 2,  /* valid request outside what this library implements */
  RA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                 */
  RA_ERR_TIMEOUT = 4       /* a bounded device-side wait gave up (see below)    */
} ra_status;

/*
 * ring_attn_fwd -- forward ring-ordered blockwise attention.
 *
 * Computes, for every batch b, query head h and row r,
 *     out[b, r, h, :] = sum_c softmax_c(scale * q[b,r,h,:] . k[b,c,h/g,:]) v[b,c,h/g,:]
 *     lse[b, h, r]    = ln sum_c exp(scale * q[b,r,h,:] . k[b,c,h/g,:])
 * over the keys c allowed by the mask (all c, or c <= r when causal), with
 * g = Hq / Hkv query heads sharing one K/V head (grouped-query attention,
 * lnwmold page §2.2; contiguous groups: head h reads K/V head h / g).  The
 * work is organised as the ring of the pages: query block i visits K/V blocks
 * (i - t) mod n_ring, t = 0..n_ring-1; causal visits with j > i are skipped,
 * the j == i visit is masked on its diagonal, j < i visits run unmasked.
 *
 *   q      bf16 [B, L, Hq,  d], contiguous (d fastest)              (in)
 *   k, v   bf16 [B, L, Hkv, d], contiguous                          (in)
 *   out    bf16 [B, L, Hq,  d], contiguous, fp32-accumulated and
 *          rounded to nearest even                                  (out)
 *   lse    fp32 [B, Hq, L], contiguous, natural-log log-sum-exp     (out)
 *   B, Hq, Hkv, L, d, n_ring   sizes; L % n_ring == 0 (equal blocks),
 *          Hq % Hkv == 0, d in {64, 128}; any block length L/n_ring >= 1
 *          (blocks that are not a multiple of 128 rows end in a partial
 *          tile); B*L < 2^31.
 *   causal 0 or 1
 *   scale  finite and >= 0 (the pages use 1/sqrt(d); 0 gives uniform weights)
 *
 * Pointers must be 16-byte aligned and out/lse must not overlap the inputs.
 * B*Hq*L == 0 is a valid empty problem: nothing is launched and the pointers
 * may be NULL.
 * Errors: RA_ERR_INVALID_ARG for the conditions above, RA_ERR_UNSUPPORTED for
 * d outside {64, 128} or a device that is not compute capability 10.0,
 * RA_ERR_CUDA if the launch fails.  Nothing is written on error.
 */
ra_status ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int Hq, int Hkv, int64_t L, int d, int n_ring, int causal,
                        float scale, ra_stream_t stream);

/*
 * ring_attn_fwd_visit -- one ring step of one host: its query block against
 * the K/V block it holds at that step, folded into its running output
 * ("Ring Attention 环注意力" L4 §4.2 steps 1-2: compute on the block in
 * hand, accumulate into O_i, pass K/V on; the striped and zigzag layouts of
 * L4 §4.5 limitation 2 and §4.8 use the same visits on other row sets).
 * A multi-device ring calls this once per step while the next K/V block is
 * in flight; the exchange itself is the caller's (the Python ring driver
 * uses torch.distributed send/recv).
 *
 * For every batch b, query head h and row r of the block (l rows):
 *     o_t[b, r, h, :] = sum_c softmax_c(scale * q[b,r,h,:] . k[b,c,h/g,:]) v[b,c,h/g,:]
 *     lse_t[b, h, r]  = ln sum_c exp(scale * q[b,r,h,:] . k[b,c,h/g,:])
 * over the keys c of the K/V block allowed by `diag`:
 *   diag == 0: all c (a block earlier in the sequence, or no causal mask);
 *   diag == 1: c <= r (the host's own block under causal masking, or, in a
 *              striped layout, a block from a host at or before this one);
 *   diag == 2: c < r (striped layout, a block from a later host: its key at
 *              local row r follows the query in the sequence).  Local row 0
 *              has no key: its partial is empty, o_t = 0 and lse_t = -inf,
 *              which the fold ignores (on the first visit o_acc row = 0,
 *              lse_acc = -inf).
 * fold == 0: o_acc = o_t, lse_acc = lse_t (the first visit).
 * fold == 1: (o_acc, lse_acc) = merge((o_acc, lse_acc), (o_t, lse_t)) with
 *   the row merge of ring_attn_merge, bitwise the same as writing o_t/lse_t
 *   to separate buffers and merging them with ring_attn_merge.
 * out, if not NULL, receives the bf16 (round to nearest even) copy of the
 * new o_acc: pass it on the last visit to get the finished output.
 *
 *   q       bf16 [B, l, Hq,  d] contiguous: the host's query block     (in)
 *   k, v    bf16 [B, l, Hkv, d] contiguous: the visited K/V block      (in)
 *   o_acc   fp32 [B, l, Hq,  d] contiguous (read when fold == 1)    (in/out)
 *   lse_acc fp32 [B, Hq, l] contiguous, natural log (read when fold) (in/out)
 *   out     bf16 [B, l, Hq,  d] contiguous, or NULL                    (out)
 *   B, Hq, Hkv, l, d   as for ring_attn_fwd with L = l, n_ring = 1.
 *   diag 0, 1 or 2; fold 0 or 1; scale finite and >= 0.
 *
 * Pointers must be 16-byte aligned; o_acc, lse_acc and out must not overlap
 * the inputs or each other.  B*Hq*l == 0 launches nothing.  Errors as for
 * ring_attn_fwd; nothing is written on an argument error.
 */
ra_status ring_attn_fwd_visit(const void* q, const void* k, const void* v, float* o_acc,
                              float* lse_acc, void* out, int B, int Hq, int Hkv, int64_t l, int d,
                              int diag, int fold, float scale, ra_stream_t stream);

/*
 * ring_attn_bwd_workspace_size -- bytes of device workspace ring_attn_bwd
 * needs: one fp32 per query row and head (B * Hq * L * 4).
 */
ra_status ring_attn_bwd_workspace_size(int B, int Hq, int64_t L, size_t* bytes);

/*
 * ring_attn_bwd -- backward pass of ring_attn_fwd: the gradients of
 * sum(out * dout) with respect to q, k and v, recomputing the attention
 * weights from the forward's lse instead of storing them (FlashAttention
 * article, section 二, 核心原理 / 重计算):
 *     P  = exp(scale * Q K^T - lse)   (masked entries 0)
 *     dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D)
 *     dQ = scale * dS K,  dK = scale * dS^T Q
 * with the K/V gradient of each grouped-query head summed over its group.
 * The work follows the ring of "Ring Attention 环注意力" L4 §4.2: the query
 * block of host i visits K/V blocks (i - t) mod n_ring and the K/V block of
 * host j (with its dK, dV) visits query blocks (j + t) mod n_ring; causal
 * visits of a later K/V block are skipped.  P and dS are rounded to bf16
 * before their products (as P is in the forward), accumulation is fp32,
 * outputs are rounded to nearest even.
 *
 *   q, k, v, scale, B, Hq, Hkv, L, d, n_ring, causal   exactly as given to
 *          ring_attn_fwd (same layouts and limits)                    (in)
 *   out    bf16 [B, L, Hq, d]: the forward output                     (in)
 *   dout   bf16 [B, L, Hq, d]: the gradient of the loss w.r.t. out     (in)
 *   lse    fp32 [B, Hq, L]: the forward lse                          (in)
 *   dq     bf16 [B, L, Hq, d]                                        (out)
 *   dk, dv bf16 [B, L, Hkv, d]                                       (out)
 *   workspace  device memory of at least ring_attn_bwd_workspace_size
 *          bytes, owned by the caller; holds D between the two kernels of
 *          the call, so two calls in flight at once need two workspaces.
 *
 * Pointers must be 16-byte aligned; outputs and workspace must not overlap
 * the inputs or each other.  B*Hq*L == 0 launches nothing.  Errors as for
 * ring_attn_fwd, plus RA_ERR_INVALID_ARG for a short workspace.  Two kernels
 * are launched on `stream` (dQ with D first, then dK/dV).
 */
ra_status ring_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                        int64_t L, int d, int n_ring, int causal, float scale,
                        ra_stream_t stream);

/*
 * ring_attn_bwd_visit -- one ring step of the backward pass on one host: its
 * query block against the K/V block it holds, adding the step's share to the
 * host's dQ accumulator and to the travelling dK, dV accumulators of that
 * K/V block (which move around the ring with K and V, as in "Ring Attention
 * 环注意力" L4 §4.2, so that every host adds its share before the block
 * returns home).  The arithmetic is ring_attn_bwd's, restricted to one
 * (query block, K/V block) pair with the mask `diag` of ring_attn_fwd_visit
 * (0 every key, 1 keys c <= r, 2 keys c < r; local rows):
 *
 *   parts & 1: D = rowsum(dout * out) of the query block into `workspace`,
 *              then dq_acc (fp32 [B, l, Hq, d]) = (fold_q ? dq_acc : 0)
 *              + scale * dS K; dq (bf16, may be NULL) gets the rounded
 *              new dq_acc.
 *   parts & 2: dk_acc, dv_acc (fp32 [B, l, Hkv, d]) = (fold_kv ? acc : 0)
 *              + scale * dS^T Q, P^T dO; reads D from `workspace`, which an
 *              earlier call with parts & 1 for the same query block (out,
 *              dout) must have written on the same stream.
 *   Both halves may be launched by one call (parts = 3), or separately so
 *   that a caller can receive the incoming dK, dV accumulators while the dQ
 *   half computes.
 *
 *   q, out, dout  bf16 [B, l, Hq, d]: the host's query block, its forward
 *                 output and the loss gradient for it                 (in)
 *   lse           fp32 [B, Hq, l]: the host's final forward lse (over the
 *                 whole sequence, not this visit)                     (in)
 *   k, v          bf16 [B, l, Hkv, d]: the visited K/V block            (in)
 *   workspace     >= B * Hq * l * 4 bytes (ring_attn_bwd_workspace_size
 *                 with L = l)                                        (in/out)
 *   B, Hq, Hkv, l, d, scale   as for ring_attn_fwd with L = l, n_ring = 1;
 *   diag 0..2; parts 1..3; fold_q, fold_kv 0 or 1.
 *
 * Pointers must be 16-byte aligned; accumulators, dq and workspace must not
 * overlap the inputs or each other.  Errors as for ring_attn_bwd.
 */
ra_status ring_attn_bwd_visit(const void* q, const void* k, const void* v, const void* out,
                              const void* dout, const float* lse, float* dq_acc, float* dk_acc,
                              float* dv_acc, void* dq, void* workspace, size_t workspace_bytes,
                              int B, int Hq, int Hkv, int64_t l, int d, int diag, int parts,
                              int fold_q, int fold_kv, float scale, ra_stream_t stream);

/*
 * ring_attn_round_bf16 -- dst[i] = src[i] rounded to bf16 (nearest even),
 * i < n: turns a travelling fp32 gradient accumulator into the bf16 result
 * once it is home.  src fp32, dst bf16, both 16-byte aligned, n % 8 == 0,
 * no overlap.  n == 0 launches nothing.
 */
ra_status ring_attn_round_bf16(const float* src, void* dst, int64_t n, ra_stream_t stream);

/*
 * ring_attn_bwd_noalloc -- ring_attn_bwd for callers that cannot allocate
 * device memory for its workspace.  The pages have no counterpart: this is
 * an interface convenience, not a step of the method.
 *
 * Who needs it: a caller whose device memory is owned by someone else (a
 * framework's caching allocator or a fixed budget reserved at start-up that
 * this library cannot draw from), or one that must not call cudaMalloc and
 * cudaFree on its hot path because cudaFree synchronises the device.  This
 * entry point allocates nothing: the D vector that ring_attn_bwd keeps in the
 * caller's workspace lives here in a fixed device array of the library
 * (4 MiB: B * Hq * L <= 1,048,576 query rows), which is part of the loaded
 * module rather than created by any allocation call.
 *
 *   Arguments, layouts, results and errors: those of ring_attn_bwd without
 *   the workspace pair; the results are bitwise those of ring_attn_bwd.
 *   B * Hq * L above 1,048,576 is rejected with RA_ERR_INVALID_ARG before
 *   anything is launched (use ring_attn_bwd with a workspace instead).
 *
 * Nothing in the fixed array has to start at zero: each call writes every
 * entry it later reads.  The array is shared by every call on a device, so
 * two calls whose kernels may run at the same time (on different streams,
 * or from different host threads) race on it and corrupt each other's
 * results: order them on one stream, or use ring_attn_bwd with a workspace
 * per concurrent call.  The array belongs to the module loaded in each CUDA
 * context.  A call made while `stream` is not capturing looks up the array's
 * address in the current context (cudaGetSymbolAddress) and remembers it for
 * that context.  A call made during a stream capture uses the remembered
 * address, so make the first call in each context before any stream capture
 * begins.
 */
ra_status ring_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                int B, int Hq, int Hkv, int64_t L, int d, int n_ring, int causal,
                                float scale, ra_stream_t stream);

/*
 * ring_attn_merge -- fold two partial attention results over disjoint key
 * sets into one (the accumulation of each ring step's blockwise result into
 * O_i, "Ring Attention 环注意力" L4 §4.2 step 2, kept as output plus
 * logsumexp as in FlashAttention-2):
 *     M = max(lse_a, lse_b), w = exp(lse - M)
 *     lse_out = M + ln(w_a + w_b)
 *     o_out   = (w_a o_a + w_b o_b) / (w_a + w_b)
 * A partial with lse = -inf is empty: the other one is returned exactly (its
 * o may hold anything, NaN included); two empty partials give o = 0 and
 * lse = -inf.  NaN in an lse propagates to that row.  The result is bitwise
 * identical when a and b are swapped.
 *
 *   o_a, o_b, o_out   fp32 [rows, d], contiguous
 *   lse_a, lse_b, lse_out fp32 [rows]
 *   rows >= 0, d >= 1 with d % 4 == 0; 16-byte aligned pointers.
 * o_out/lse_out may be exactly o_a/lse_a or o_b/lse_b (in place); any other
 * overlap is invalid.  rows == 0 launches nothing.
 */
ra_status ring_attn_merge(const float* o_a, const float* lse_a, const float* o_b,
                          const float* lse_b, float* o_out, float* lse_out, int64_t rows, int d,
                          ra_stream_t stream);

/*
 * ring_attn_quantize_fp8 -- block quantisation of a bf16 tensor to E4M3 for
 * ring_attn_fwd_fp8 (the FP8 forward of the FlashAttention article,
 * developer.aliyun page, section 二, FlashAttention-3: FP8 GEMMs with block
 * quantisation).  A block is the 128-row tile of one (batch, head):
 *     scale[b, h, t] = amax / 448 in float32 (1 if the tile is all zeros),
 *                      amax over rows [128t, 128t + 128) and all d columns;
 *     codes[b, r, h, c] = E4M3(x[b, r, h, c] / scale), the quotient rounded
 *                      to float32, then to E4M3 (OCP 8-bit format: bias 7,
 *                      largest finite 448, no infinities) with ties to even,
 *                      magnitudes above 448 saturated.
 * When L is not a multiple of 128 the last tile holds the remaining rows.
 *
 *   x       bf16 [B, L, H, d], contiguous, 16-byte aligned, finite values
 *   codes   uint8 [B, L, H, d] (E4M3 bit patterns), 16-byte aligned
 *   scales  fp32 [B, H, ceil(L / 128)], 4-byte aligned
 *   d a multiple of 8 in [8, 256]; B, H <= 65535.  Outputs must not overlap x
 *   or each other.  B*H*L == 0 launches nothing.
 * Errors: RA_ERR_INVALID_ARG for negative sizes, null, misaligned or
 * overlapping pointers; RA_ERR_UNSUPPORTED for other d or B, H above 65535.
 */
ra_status ring_attn_quantize_fp8(const void* x, void* codes, float* scales, int B, int64_t L,
                                 int H, int d, ra_stream_t stream);

/*
 * ring_attn_fwd_fp8 -- the ring-ordered forward of ring_attn_fwd (same
 * blocks, ring order, causal skipping and masking, GQA mapping and lse
 * convention) computed from block-quantised E4M3 inputs: both GEMMs on the
 * FP8 tensor cores, scores scaled by scale * sq * sk per tile pair, fp32
 * softmax statistics, the probabilities rounded to E4M3 before the P V
 * product, bf16 output.  It approximates exact attention of the dequantised
 * tensors code * scale; the error is that of E4M3 probabilities (relative
 * 2^-4 per weight, absolute 2^-10 below E4M3's normal range).
 *
 *   q8            uint8 [B, L, Hq, 128]  E4M3 codes (ring_attn_quantize_fp8)
 *   k8, v8        uint8 [B, L, Hkv, 128]
 *   sq            fp32 [B, Hq, L / 128]  tile scales, finite and > 0
 *   sk, sv        fp32 [B, Hkv, L / 128]
 *   out           bf16 [B, L, Hq, 128]
 *   lse           fp32 [B, Hq, L], natural log
 *   d must be 128 and L / n_ring a multiple of 128 (else RA_ERR_UNSUPPORTED);
 *   the other sizes, values and errors are those of ring_attn_fwd.  All
 *   pointers 16-byte aligned; outputs must not overlap the inputs or each
 *   other.
 */
ra_status ring_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                            const float* sk, const float* sv, void* out, float* lse, int B, int Hq,
                            int Hkv, int64_t L, int d, int n_ring, int causal, float scale,
                            ra_stream_t stream);

/*
 * ring_attn_check_status -- synchronise `stream`, then read and clear the
 * device status words of the current device.  Every device-side wait of the
 * forward (bf16 and FP8) and backward kernels is bounded (see
 * ring_attn_set_wait_limit_ns); a wait that
 * runs out makes the kernel record RA_ERR_TIMEOUT, release its tensor memory
 * and return, leaving the CUDA context usable.  Returns RA_ERR_CUDA if the
 * synchronisation itself fails.
 */
ra_status ring_attn_check_status(ra_stream_t stream);

/* Longest any single device-side wait may take before the kernel gives up
 * (nanoseconds; default 5e9).  0 restores the default.  Process-wide. */
ra_status ring_attn_set_wait_limit_ns(uint64_t ns);

/* Cap on the number of persistent CTAs of the forward and backward kernels
 * (0 = one per SM, the default).  Process-wide; used to exercise the
 * scheduler.  Results do not depend on it. */
ra_status ring_attn_set_max_ctas(int n);

/* Order in which the forward kernels' persistent CTAs (bf16 and FP8) take
 * work units from the launch's queue (a unit = two 128-row query tiles
 * sharing one K/V stream; causal units differ in length).  Results do not
 * depend on it.  Process-wide.
 *   RA_SCHEDULE_AUTO (default): HEAD_MAJOR when the K/V tensors exceed
 *     96 MiB, else LONGEST_FIRST.
 *   RA_SCHEDULE_LONGEST_FIRST: every unit sorted by length, longest first
 *     (causal load balance, "Ring Attention 环注意力" L4 §4.5 limitation 3).
 *   RA_SCHEDULE_HEAD_MAJOR: longest first within each (batch, K/V head), heads
 *     one after another, so concurrently running CTAs share K/V tiles in L2. */
enum { RA_SCHEDULE_AUTO = 0, RA_SCHEDULE_LONGEST_FIRST = 1, RA_SCHEDULE_HEAD_MAJOR = 2 };
ra_status ring_attn_set_schedule(int schedule);

/* Host-side fault injection for tests.  Bit 0: the loader of the forward
 * kernels (bf16 and FP8) and of the backward dQ kernel skips its first
 * query-tile load, so
 * the first bounded wait on it runs out and the call reports RA_ERR_TIMEOUT
 * through ring_attn_check_status.  0 clears.  Process-wide. */
ra_status ring_attn_debug_inject(unsigned flags);

/* Human-readable name of a status code (static storage). */
const char* ring_attn_status_string(ra_status s);

/* Explanation of the last non-OK status returned on this host thread
 * ("" if none).  Valid until the next call on the same thread. */
const char* ring_attn_last_error(void);

/* Library ABI version (major * 100 + minor). */
int ring_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RING_ATTN_H_ */
