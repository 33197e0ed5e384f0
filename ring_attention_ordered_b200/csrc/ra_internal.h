// Internal declarations shared by the kernels and the C ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace ra {

// Parameters of one forward launch.  The tensor maps describe q, k and v as
// 3-D arrays {d, H, B*L} of bf16 (d fastest) with a box of {64, 1, 128}:
// 64 head-dim columns (one 128-byte swizzle row) of 128 consecutive rows of
// one head.
struct FwdParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  __nv_bfloat16* out;  // bf16 output; may be NULL in a per-visit launch
  float* lse;
  // Per-visit launch (o_acc != NULL): the whole launch is one ring visit of a
  // query block against one K/V block (n_ring == 1, causal == diagonal
  // visit); its fp32 result goes to o_acc [B, L, Hq, d] and lse, folded into
  // what they hold when visit_fold == 1, and out (if not NULL) receives the
  // bf16 rounding of the folded result.
  float* o_acc;
  int visit_fold;
  int diag_shift;      // 1: the diagonal visit excludes the key at the query's own row
  int B, Hq, Hkv, group;
  int L, blk_len, n_ring, causal;
  int tiles_per_blk;   // ceil(blk_len / 128)
  int pair_heads;      // 1: a unit is two heads of one GQA group on the same rows
  int head_slots;      // ceil(group / 2), when pair_heads
  int pairs_per_blk;   // ceil(tiles_per_blk / 2), when !pair_heads
  int total_units;     // < 2^31, checked by the host
  int head_major;      // unit order: 1 = K/V-head major (L2 reuse), 0 = global longest first
  float scale_log2;    // scale * log2(e)
  unsigned long long wait_limit_ns;
  unsigned debug_flags;
  // Work queue of this launch: a counter (zero at launch) from which each
  // CTA's loader takes the next unit, in the unit order above.
  unsigned int* tickets;
};

// Parameters of one FP8 forward launch (d = 128).  The tensor maps describe
// the E4M3 codes of q, k and v as 3-D byte arrays {128, H, B*L} with a box of
// {128, 1, 128}: one 128-byte swizzle row per head row, 128 consecutive rows
// of one head.  sq [B, Hq, T], sk and sv [B, Hkv, T] hold the float32 scale
// of each 128-row tile (T = L / 128).  The scheduling fields mean what they
// mean in FwdParams.
struct Fp8FwdParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const float* sq;
  const float* sk;
  const float* sv;
  __nv_bfloat16* out;
  float* lse;
  int B, Hq, Hkv, group;
  int L, blk_len, n_ring, causal;
  int tiles_per_blk;
  int pair_heads;
  int head_slots;
  int pairs_per_blk;
  int total_units;
  int head_major;
  int n_tiles;         // T = L / 128
  float scale_log2;    // scale * log2(e), before the per-tile scales
  unsigned long long wait_limit_ns;
  unsigned debug_flags;
  unsigned int* tickets;   // the launch's work queue (see FwdParams)
};

// Parameters of the two backward launches (dQ kernel, then dK/dV kernel).
// tm_q/tm_do view q and dout as {d, Hq, B*L}, tm_k/tm_v view k and v as
// {d, Hkv, B*L}, with the forward's box and swizzle.
struct BwdParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_do;
  const __nv_bfloat16* out;    // forward output O [B, L, Hq, d]
  const __nv_bfloat16* dout;   // upstream gradient dO [B, L, Hq, d]
  const float* lse;            // forward lse [B, Hq, L] (natural log)
  float* dvec;                 // workspace: D = rowsum(dO * O) [B, Hq, L]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int B, Hq, Hkv, group;
  int L, blk_len, n_ring, causal;
  int tiles_per_blk;
  int units_dq;                // B * Hq * n_ring * tiles_per_blk
  int units_kv;                // B * Hkv * n_ring * tiles_per_blk
  // work-queue counters of the two launches (set by the launcher, see
  // next_ticket_counter)
  unsigned int* tickets_dq;
  unsigned int* tickets_kv;
  float scale;
  float scale_log2;
  unsigned long long wait_limit_ns;
  unsigned debug_flags;
  // Which kernels run: bit 0 the dQ kernel (also writes D), bit 1 the dK/dV
  // kernel (reads D).  ring_attn_bwd runs both.
  int parts;
  // Per-visit launches (ring_attn_bwd_visit): when dq_acc / dk_acc are set,
  // the dQ (dK, dV) rows are written to, or with fold_q (fold_kv) added to,
  // these fp32 accumulators [B, L, H, d]; dq, if set, then receives the bf16
  // rounding of the new dq_acc.  diag_shift = 1 makes the diagonal block
  // exclude the key at the query's own row.
  float* dq_acc;
  float* dk_acc;
  float* dv_acc;
  int fold_q, fold_kv;
  int diag_shift;
};

cudaError_t launch_fwd(const FwdParams& prm, int d, int grid, cudaStream_t stream);
cudaError_t launch_bwd(const BwdParams& prm, int d, int num_sms, int max_ctas,
                       cudaStream_t stream);
cudaError_t read_and_clear_bwd_status(unsigned long long* out);

// Static scratch of ring_attn_bwd_noalloc (fp32 entries, 4 MiB).
constexpr long long kNoAllocScratchRows = 1ll << 20;
// Device address of that scratch in the current context.  Looked up on every
// call made while `stream` is not capturing (the module, and so the address,
// belongs to a context, which cudaDeviceReset or a caller's own context can
// change); during a capture the address cached for the current context is
// used, so a context's first call must come before any capture.
cudaError_t noalloc_scratch(void** ptr, cudaStream_t stream);
// The calling thread's current driver context (nullptr if none).
cudaError_t current_context(CUcontext* ctx);
// Device address of a static __device__ variable of this library in the
// current context.  Looked up on every call made while `stream` is not
// capturing (the module, and so the address, belongs to a context, which
// cudaDeviceReset or a caller's own context can change); during a capture
// the address last found for the current context is used.
cudaError_t symbol_address(const void* symbol, void** ptr, cudaStream_t stream);
cudaError_t read_and_clear_status(unsigned long long* out);
// A zeroed work-queue counter for the next launch on `stream` (forward, FP8
// forward, each backward kernel): one of kTicketSlots static device
// counters, taken in rotation and reset by a memset ordered on the stream
// (so launches on different streams use different counters, up to
// kTicketSlots at a time).
constexpr int kTicketSlots = 64;
cudaError_t next_ticket_counter(cudaStream_t stream, unsigned int** counter);

cudaError_t launch_fwd_fp8(const Fp8FwdParams& prm, int grid, cudaStream_t stream);
cudaError_t read_and_clear_fp8_status(unsigned long long* out);
// Block quantisation of x bf16 [B, L, H, d] to E4M3 codes and per-tile scales.
cudaError_t launch_quantize_fp8(const __nv_bfloat16* x, uint8_t* codes, float* scales, int B,
                                long long L, int H, int d, cudaStream_t stream);

cudaError_t launch_round_bf16(const float* src, __nv_bfloat16* dst, long long n, int num_sms,
                              cudaStream_t stream);

cudaError_t launch_merge(const float* o_a, const float* lse_a, const float* o_b,
                         const float* lse_b, float* o_out, float* lse_out, long long rows, int d,
                         int num_sms, cudaStream_t stream);

}  // namespace ra
