// C ABI of libring_attn: argument validation, TMA tensor-map construction,
// work-unit planning and launches.  Declared in include/ring_attn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "ra_internal.h"
#include "ring_attn.h"

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_wait_limit_ns{5000000000ull};
std::atomic<int> g_max_ctas{0};
std::atomic<unsigned> g_debug_flags{0u};
// Work-unit order: RA_SCHEDULE_AUTO picks K/V-head-major order when the K/V
// tensors are larger than about 3/4 of L2 (CTAs then share one or two K/V
// heads at a time, which stay L2-resident), else global longest-first order
// (best load balance when K/V fits L2 anyway).  Measured with the work
// queue: head-major is 1-2% faster at 128 MiB of K/V (the 32K GQA case) and
// 23% slower at 64 MiB (the 8K case, whose 16 heads then run a few at a time
// with short units).
std::atomic<int> g_schedule{RA_SCHEDULE_AUTO};
constexpr double kHeadMajorKvBytes = 96.0 * 1024 * 1024;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
int g_cc_ok[kMaxDevices] = {0};  // 0 unknown, 1 yes, -1 no
std::mutex g_mu;

ra_status fail(ra_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

ra_status ok() {
  g_last_error.clear();
  return RA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace ra {

// The calling thread's current driver context (nullptr if none), through the
// driver entry point the runtime exposes (no link against libcuda).
cudaError_t current_context(CUcontext* ctx) {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  if (!fn) return cudaErrorNotSupported;
  *ctx = nullptr;
  return fn(ctx) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

cudaError_t symbol_address(const void* symbol, void** ptr, cudaStream_t stream) {
  struct Entry {
    CUcontext ctx;
    const void* symbol;
    void* addr;
  };
  static std::mutex mu;
  static Entry cache[64] = {};
  static int n_cached = 0;
  CUcontext ctx = nullptr;
  cudaError_t e = current_context(&ctx);
  if (e != cudaSuccess) return e;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  int slot = -1;
  for (int i = 0; i < n_cached; ++i)
    if (cache[i].ctx == ctx && cache[i].symbol == symbol) slot = i;
  if (cs == cudaStreamCaptureStatusNone || slot < 0 || ctx == nullptr) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, symbol);
    if (e != cudaSuccess) return e;
    // the lookup made a context current if there was none
    if (ctx == nullptr && (e = current_context(&ctx)) != cudaSuccess) return e;
    for (int i = 0; i < n_cached; ++i)
      if (cache[i].ctx == ctx && cache[i].symbol == symbol) slot = i;
    if (slot < 0) slot = (n_cached < 64) ? n_cached++ : 0;
    cache[slot] = Entry{ctx, symbol, addr};
  }
  *ptr = cache[slot].addr;
  return cudaSuccess;
}

}  // namespace ra

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Query SM count and compute capability of the current device once.  A
// thread with no current context (one that has only been told its device,
// such as torch's autograd worker) gets the device's primary context made
// current, since the tensor-map encoder needs a context; a context the caller
// made current itself (primary or its own, cuCtxCreate) is left in place and
// used.
ra_status device_info(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(RA_ERR_UNSUPPORTED, "device index %d", dev);
  CUcontext cur = nullptr;
  if ((e = ra::current_context(&cur)) != cudaSuccess)
    return fail(RA_ERR_CUDA, "cuCtxGetCurrent: %s", cudaGetErrorString(e));
  if (cur == nullptr && (e = cudaSetDevice(dev)) != cudaSuccess)
    return fail(RA_ERR_CUDA, "cudaSetDevice: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_cc_ok[dev] == 0) {
    int major = 0, minor = 0, n = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return fail(RA_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    g_cc_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    g_sm_count[dev] = n;
  }
  if (g_cc_ok[dev] != 1)
    return fail(RA_ERR_UNSUPPORTED, "this library is built for sm_100a (compute capability 10.0)");
  *sms = g_sm_count[dev];
  return RA_OK;
}

// Tensor map over a bf16 [B*L, H, d] array (d fastest): box {64, 1, 128},
// 128-byte swizzle, out-of-range rows read as zero.
ra_status make_map(CUtensorMap* map, const void* base, int H, long long rows, int d) {
  auto enc = get_encode_fn();
  if (!enc) return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return RA_OK;
}

// Tensor map over the E4M3 codes of a [B*L, H, 128] byte array: box
// {128, 1, 128} (one 128-byte swizzle row per head row), 128-byte swizzle.
ra_status make_map_e4m3(CUtensorMap* map, const void* base, int H, long long rows) {
  auto enc = get_encode_fn();
  if (!enc) return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(H) * 128};
  cuuint32_t box[3] = {128, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return RA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Shared by ring_attn_fwd and ring_attn_fwd_visit: tensor maps, work units,
// schedule and launch of the forward kernel.  Arguments are already checked.
ra_status launch_forward(const void* q, const void* k, const void* v, void* out, float* lse,
                         float* o_acc, int visit_fold, int diag_shift, int B, int Hq, int Hkv, int64_t L, int d,
                         int n_ring, int causal, float scale, size_t nkv, ra_stream_t stream) {
  int sms = 0;
  ra_status st = device_info(&sms);
  if (st != RA_OK) return st;

  ra::FwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const long long rows = static_cast<long long>(B) * L;
  if ((st = make_map(&prm.tm_q, q, Hq, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_k, k, Hkv, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_v, v, Hkv, rows, d)) != RA_OK) return st;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.o_acc = o_acc;
  prm.visit_fold = visit_fold;
  prm.diag_shift = diag_shift;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.L = static_cast<int>(L);
  prm.n_ring = n_ring;
  prm.blk_len = static_cast<int>(L / n_ring);
  prm.causal = causal;
  prm.tiles_per_blk = (prm.blk_len + 127) / 128;
  prm.pair_heads = prm.group >= 2 ? 1 : 0;
  prm.head_slots = (prm.group + 1) / 2;
  prm.pairs_per_blk = (prm.tiles_per_blk + 1) / 2;
  const long long units =
      prm.pair_heads
          ? static_cast<long long>(B) * Hkv * prm.head_slots * n_ring * prm.tiles_per_blk
          : static_cast<long long>(B) * Hq * n_ring * prm.pairs_per_blk;
  if (units >= (1ll << 31)) return fail(RA_ERR_INVALID_ARG, "problem too large (%lld work units)", units);
  prm.total_units = static_cast<int>(units);
  const int sched = g_schedule.load();
  prm.head_major = sched == RA_SCHEDULE_HEAD_MAJOR ||
                   (sched == RA_SCHEDULE_AUTO && 2.0 * static_cast<double>(nkv) > kHeadMajorKvBytes);
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  prm.wait_limit_ns = g_wait_limit_ns.load();
  prm.debug_flags = g_debug_flags.load();

  long long grid = sms;
  const int cap = g_max_ctas.load();
  if (cap > 0 && cap < grid) grid = cap;
  if (grid > prm.total_units) grid = prm.total_units;
  cudaError_t e = ra::next_ticket_counter(reinterpret_cast<cudaStream_t>(stream), &prm.tickets);
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "work queue reset: %s", cudaGetErrorString(e));
  e = ra::launch_fwd(prm, d, static_cast<int>(grid), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "forward launch: %s", cudaGetErrorString(e));
  return ok();
}

// Checks common to both forward entry points (sizes, values, head dim).
ra_status check_forward_shape(int B, int Hq, int Hkv, int64_t L, int d, int n_ring, int causal,
                              float scale) {
  if (B < 0 || Hq < 0 || Hkv < 0 || L < 0)
    return fail(RA_ERR_INVALID_ARG, "negative size (B=%d Hq=%d Hkv=%d L=%lld)", B, Hq, Hkv,
                static_cast<long long>(L));
  if (n_ring < 1) return fail(RA_ERR_INVALID_ARG, "n_ring must be >= 1 (got %d)", n_ring);
  if (causal != 0 && causal != 1) return fail(RA_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!std::isfinite(scale) || scale < 0.f)
    return fail(RA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (L % n_ring != 0)
    return fail(RA_ERR_INVALID_ARG, "L=%lld does not split into %d equal blocks",
                static_cast<long long>(L), n_ring);
  if (Hkv == 0 && Hq != 0) return fail(RA_ERR_INVALID_ARG, "Hkv must be >= 1");
  if (Hkv > 0 && Hq % Hkv != 0)
    return fail(RA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  if (d != 64 && d != 128) return fail(RA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (static_cast<long long>(B) * Hq * L != 0 && static_cast<long long>(B) * L >= (1ll << 31))
    return fail(RA_ERR_INVALID_ARG, "B*L must be < 2^31");
  return RA_OK;
}

}  // namespace

extern "C" {

ra_status ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                        int Hq, int Hkv, int64_t L, int d, int n_ring, int causal, float scale,
                        ra_stream_t stream) {
  ra_status st = check_forward_shape(B, Hq, Hkv, L, d, n_ring, causal, scale);
  if (st != RA_OK) return st;
  if (static_cast<long long>(B) * Hq * L == 0) return ok();
  if (!q || !k || !v || !out || !lse) return fail(RA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(RA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t nq = static_cast<size_t>(B) * L * Hq * d * 2;
  const size_t nkv = static_cast<size_t>(B) * L * Hkv * d * 2;
  const size_t nl = static_cast<size_t>(B) * Hq * L * 4;
  if (overlaps(out, nq, q, nq) || overlaps(out, nq, k, nkv) || overlaps(out, nq, v, nkv) ||
      overlaps(lse, nl, q, nq) || overlaps(lse, nl, k, nkv) || overlaps(lse, nl, v, nkv) ||
      overlaps(out, nq, lse, nl))
    return fail(RA_ERR_INVALID_ARG, "outputs overlap the inputs or each other");
  return launch_forward(q, k, v, out, lse, nullptr, 0, 0, B, Hq, Hkv, L, d, n_ring, causal, scale,
                        nkv, stream);
}

ra_status ring_attn_fwd_visit(const void* q, const void* k, const void* v, float* o_acc,
                              float* lse_acc, void* out, int B, int Hq, int Hkv, int64_t l, int d,
                              int diag, int fold, float scale, ra_stream_t stream) {
  if (diag < 0 || diag > 2) return fail(RA_ERR_INVALID_ARG, "diag must be 0, 1 or 2");
  if (fold != 0 && fold != 1) return fail(RA_ERR_INVALID_ARG, "fold must be 0 or 1");
  ra_status st = check_forward_shape(B, Hq, Hkv, l, d, 1, diag != 0, scale);
  if (st != RA_OK) return st;
  if (static_cast<long long>(B) * Hq * l == 0) return ok();
  if (!q || !k || !v || !o_acc || !lse_acc) return fail(RA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_acc) || !aligned16(lse_acc) ||
      !aligned16(out))
    return fail(RA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t nq = static_cast<size_t>(B) * l * Hq * d * 2;
  const size_t nkv = static_cast<size_t>(B) * l * Hkv * d * 2;
  const size_t no = 2 * nq;
  const size_t nl = static_cast<size_t>(B) * Hq * l * 4;
  const void* ins[3] = {q, k, v};
  const size_t in_n[3] = {nq, nkv, nkv};
  for (int i = 0; i < 3; ++i)
    if (overlaps(o_acc, no, ins[i], in_n[i]) || overlaps(lse_acc, nl, ins[i], in_n[i]) ||
        (out && overlaps(out, nq, ins[i], in_n[i])))
      return fail(RA_ERR_INVALID_ARG, "outputs overlap the inputs");
  if (overlaps(o_acc, no, lse_acc, nl) || (out && (overlaps(out, nq, o_acc, no) ||
                                                   overlaps(out, nq, lse_acc, nl))))
    return fail(RA_ERR_INVALID_ARG, "o_acc, lse_acc and out overlap each other");
  return launch_forward(q, k, v, out, lse_acc, o_acc, fold, diag == 2, B, Hq, Hkv, l, d, 1,
                        diag != 0, scale, nkv, stream);
}

ra_status ring_attn_bwd_workspace_size(int B, int Hq, int64_t L, size_t* bytes) {
  if (!bytes) return fail(RA_ERR_INVALID_ARG, "null size pointer");
  if (B < 0 || Hq < 0 || L < 0) return fail(RA_ERR_INVALID_ARG, "negative size");
  *bytes = static_cast<size_t>(B) * static_cast<size_t>(Hq) * static_cast<size_t>(L) * 4;
  return ok();
}

ra_status ring_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                        int64_t L, int d, int n_ring, int causal, float scale,
                        ra_stream_t stream) {
  ra_status st = check_forward_shape(B, Hq, Hkv, L, d, n_ring, causal, scale);
  if (st != RA_OK) return st;
  if (static_cast<long long>(B) * Hq * L == 0) return ok();
  const size_t nq = static_cast<size_t>(B) * L * Hq * d * 2;
  const size_t nkv = static_cast<size_t>(B) * L * Hkv * d * 2;
  const size_t nl = static_cast<size_t>(B) * Hq * L * 4;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !workspace)
    return fail(RA_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[10] = {q, k, v, out, dout, lse, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return fail(RA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (workspace_bytes < nl)
    return fail(RA_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu needed",
                workspace_bytes, nl);
  const void* ins[6] = {q, k, v, out, dout, lse};
  const size_t in_n[6] = {nq, nkv, nkv, nq, nq, nl};
  const void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_n[4] = {nq, nkv, nkv, nl};
  for (int o = 0; o < 4; ++o) {
    for (int i = 0; i < 6; ++i)
      if (overlaps(outs[o], out_n[o], ins[i], in_n[i]))
        return fail(RA_ERR_INVALID_ARG, "an output or the workspace overlaps an input");
    for (int o2 = o + 1; o2 < 4; ++o2)
      if (overlaps(outs[o], out_n[o], outs[o2], out_n[o2]))
        return fail(RA_ERR_INVALID_ARG, "outputs and workspace overlap each other");
  }
  int sms = 0;
  if ((st = device_info(&sms)) != RA_OK) return st;
  ra::BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const long long rows = static_cast<long long>(B) * L;
  if ((st = make_map(&prm.tm_q, q, Hq, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_k, k, Hkv, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_v, v, Hkv, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_do, dout, Hq, rows, d)) != RA_OK) return st;
  prm.out = static_cast<const __nv_bfloat16*>(out);
  prm.dout = static_cast<const __nv_bfloat16*>(dout);
  prm.lse = lse;
  prm.dvec = static_cast<float*>(workspace);
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.L = static_cast<int>(L);
  prm.n_ring = n_ring;
  prm.blk_len = static_cast<int>(L / n_ring);
  prm.causal = causal;
  prm.tiles_per_blk = (prm.blk_len + 127) / 128;
  const long long uq = static_cast<long long>(B) * Hq * n_ring * prm.tiles_per_blk;
  const long long ukv = static_cast<long long>(B) * Hkv * n_ring * prm.tiles_per_blk;
  if (uq >= (1ll << 31)) return fail(RA_ERR_INVALID_ARG, "problem too large (%lld work units)", uq);
  prm.units_dq = static_cast<int>(uq);
  prm.units_kv = static_cast<int>(ukv);
  prm.scale = scale;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  prm.wait_limit_ns = g_wait_limit_ns.load();
  prm.debug_flags = g_debug_flags.load();
  prm.parts = 3;
  cudaError_t e = ra::launch_bwd(prm, d, sms, g_max_ctas.load(),
                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "backward launch: %s", cudaGetErrorString(e));
  return ok();
}

ra_status ring_attn_bwd_visit(const void* q, const void* k, const void* v, const void* out,
                              const void* dout, const float* lse, float* dq_acc, float* dk_acc,
                              float* dv_acc, void* dq, void* workspace, size_t workspace_bytes,
                              int B, int Hq, int Hkv, int64_t l, int d, int diag, int parts,
                              int fold_q, int fold_kv, float scale, ra_stream_t stream) {
  if (diag < 0 || diag > 2) return fail(RA_ERR_INVALID_ARG, "diag must be 0, 1 or 2");
  if (parts < 1 || parts > 3) return fail(RA_ERR_INVALID_ARG, "parts must be 1, 2 or 3");
  if ((fold_q != 0 && fold_q != 1) || (fold_kv != 0 && fold_kv != 1))
    return fail(RA_ERR_INVALID_ARG, "fold flags must be 0 or 1");
  ra_status st = check_forward_shape(B, Hq, Hkv, l, d, 1, diag != 0, scale);
  if (st != RA_OK) return st;
  if (static_cast<long long>(B) * Hq * l == 0) return ok();
  const size_t nq = static_cast<size_t>(B) * l * Hq * d * 2;
  const size_t nkv = static_cast<size_t>(B) * l * Hkv * d * 2;
  const size_t nl = static_cast<size_t>(B) * Hq * l * 4;
  if (!q || !k || !v || !out || !dout || !lse || !workspace)
    return fail(RA_ERR_INVALID_ARG, "null pointer");
  if ((parts & 1) && !dq_acc) return fail(RA_ERR_INVALID_ARG, "dq_acc is needed for the dQ part");
  if ((parts & 2) && (!dk_acc || !dv_acc))
    return fail(RA_ERR_INVALID_ARG, "dk_acc and dv_acc are needed for the dK/dV part");
  const void* ptrs[11] = {q, k, v, out, dout, lse, workspace, dq_acc, dk_acc, dv_acc, dq};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(RA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (workspace_bytes < nl)
    return fail(RA_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu needed",
                workspace_bytes, nl);
  const void* ins[6] = {q, k, v, out, dout, lse};
  const size_t in_n[6] = {nq, nkv, nkv, nq, nq, nl};
  const void* outs[5] = {workspace, (parts & 1) ? dq_acc : nullptr, (parts & 1) ? dq : nullptr,
                         (parts & 2) ? dk_acc : nullptr, (parts & 2) ? dv_acc : nullptr};
  const size_t out_n[5] = {nl, 2 * nq, nq, 2 * nkv, 2 * nkv};
  for (int o = 0; o < 5; ++o) {
    if (!outs[o]) continue;
    for (int i = 0; i < 6; ++i)
      if (overlaps(outs[o], out_n[o], ins[i], in_n[i]))
        return fail(RA_ERR_INVALID_ARG, "an output or the workspace overlaps an input");
    for (int o2 = o + 1; o2 < 5; ++o2)
      if (outs[o2] && overlaps(outs[o], out_n[o], outs[o2], out_n[o2]))
        return fail(RA_ERR_INVALID_ARG, "outputs and workspace overlap each other");
  }
  int sms = 0;
  if ((st = device_info(&sms)) != RA_OK) return st;
  ra::BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const long long rows = static_cast<long long>(B) * l;
  if ((st = make_map(&prm.tm_q, q, Hq, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_k, k, Hkv, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_v, v, Hkv, rows, d)) != RA_OK) return st;
  if ((st = make_map(&prm.tm_do, dout, Hq, rows, d)) != RA_OK) return st;
  prm.out = static_cast<const __nv_bfloat16*>(out);
  prm.dout = static_cast<const __nv_bfloat16*>(dout);
  prm.lse = lse;
  prm.dvec = static_cast<float*>(workspace);
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.L = static_cast<int>(l);
  prm.n_ring = 1;
  prm.blk_len = static_cast<int>(l);
  prm.causal = diag != 0;
  prm.tiles_per_blk = (prm.blk_len + 127) / 128;
  const long long uq = static_cast<long long>(B) * Hq * prm.tiles_per_blk;
  if (uq >= (1ll << 31)) return fail(RA_ERR_INVALID_ARG, "problem too large (%lld work units)", uq);
  prm.units_dq = static_cast<int>(uq);
  prm.units_kv = static_cast<int>(static_cast<long long>(B) * Hkv * prm.tiles_per_blk);
  prm.scale = scale;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  prm.wait_limit_ns = g_wait_limit_ns.load();
  prm.debug_flags = g_debug_flags.load();
  prm.parts = parts;
  prm.dq_acc = dq_acc;
  prm.dk_acc = dk_acc;
  prm.dv_acc = dv_acc;
  prm.fold_q = fold_q;
  prm.fold_kv = fold_kv;
  prm.diag_shift = diag == 2;
  cudaError_t e = ra::launch_bwd(prm, d, sms, g_max_ctas.load(),
                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "backward visit launch: %s", cudaGetErrorString(e));
  return ok();
}

ra_status ring_attn_round_bf16(const float* src, void* dst, int64_t n, ra_stream_t stream) {
  if (n < 0) return fail(RA_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return ok();
  if (!src || !dst) return fail(RA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(src) || !aligned16(dst) || n % 8 != 0)
    return fail(RA_ERR_INVALID_ARG, "pointers must be 16-byte aligned and n a multiple of 8");
  if (overlaps(src, static_cast<size_t>(n) * 4, dst, static_cast<size_t>(n) * 2))
    return fail(RA_ERR_INVALID_ARG, "dst overlaps src");
  int sms = 0;
  ra_status st = device_info(&sms);
  if (st != RA_OK) return st;
  cudaError_t e = ra::launch_round_bf16(src, static_cast<__nv_bfloat16*>(dst), n, sms,
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "round launch: %s", cudaGetErrorString(e));
  return ok();
}

ra_status ring_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                int B, int Hq, int Hkv, int64_t L, int d, int n_ring, int causal,
                                float scale, ra_stream_t stream) {
  if (B < 0 || Hq < 0 || L < 0)
    return fail(RA_ERR_INVALID_ARG, "negative size (B=%d Hq=%d L=%lld)", B, Hq,
                static_cast<long long>(L));
  const long long rows = static_cast<long long>(B) * Hq * L;
  if (rows > ra::kNoAllocScratchRows)
    return fail(RA_ERR_INVALID_ARG,
                "B*Hq*L = %lld query rows exceed the %lld rows (%lld bytes) of static scratch "
                "of ring_attn_bwd_noalloc; use ring_attn_bwd with a workspace",
                rows, ra::kNoAllocScratchRows, ra::kNoAllocScratchRows * 4);
  if (rows == 0)
    return ring_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, nullptr, 0, B, Hq, Hkv, L, d,
                         n_ring, causal, scale, stream);
  void* scratch = nullptr;
  cudaError_t e = ra::noalloc_scratch(&scratch, stream);
  if (e != cudaSuccess)
    return fail(RA_ERR_CUDA, "static scratch lookup: %s", cudaGetErrorString(e));
  return ring_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, scratch,
                       static_cast<size_t>(ra::kNoAllocScratchRows) * 4, B, Hq, Hkv, L, d, n_ring,
                       causal, scale, stream);
}

ra_status ring_attn_merge(const float* o_a, const float* lse_a, const float* o_b,
                          const float* lse_b, float* o_out, float* lse_out, int64_t rows, int d,
                          ra_stream_t stream) {
  if (rows < 0) return fail(RA_ERR_INVALID_ARG, "rows must be >= 0");
  if (d < 1 || d % 4 != 0) return fail(RA_ERR_INVALID_ARG, "d must be a positive multiple of 4");
  if (rows == 0) return ok();
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out)
    return fail(RA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(o_out) || !aligned16(lse_a) ||
      !aligned16(lse_b) || !aligned16(lse_out))
    return fail(RA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t no = static_cast<size_t>(rows) * d * 4, nl = static_cast<size_t>(rows) * 4;
  auto bad_alias = [&](const void* out, size_t n, const void* in) {
    return out != in && overlaps(out, n, in, n);
  };
  if (bad_alias(o_out, no, o_a) || bad_alias(o_out, no, o_b) || bad_alias(lse_out, nl, lse_a) ||
      bad_alias(lse_out, nl, lse_b) || overlaps(o_out, no, lse_out, nl) ||
      overlaps(o_out, no, lse_a, nl) || overlaps(o_out, no, lse_b, nl) ||
      overlaps(lse_out, nl, o_a, no) || overlaps(lse_out, nl, o_b, no))
    return fail(RA_ERR_INVALID_ARG, "outputs may alias an input exactly but not overlap otherwise");
  int sms = 0;
  ra_status st = device_info(&sms);
  if (st != RA_OK) return st;
  cudaError_t e = ra::launch_merge(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d, sms,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
  return ok();
}

ra_status ring_attn_quantize_fp8(const void* x, void* codes, float* scales, int B, int64_t L,
                                 int H, int d, ra_stream_t stream) {
  if (B < 0 || H < 0 || L < 0) return fail(RA_ERR_INVALID_ARG, "negative size");
  if (d < 8 || d > 256 || d % 8 != 0)
    return fail(RA_ERR_UNSUPPORTED, "head dim %d (supported: multiples of 8 up to 256)", d);
  if (static_cast<long long>(B) * H * L == 0) return ok();
  if (B > 65535 || H > 65535) return fail(RA_ERR_UNSUPPORTED, "B and H must be <= 65535");
  if (!x || !codes || !scales) return fail(RA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return fail(RA_ERR_INVALID_ARG, "x and codes must be 16-byte aligned, scales 4-byte aligned");
  const size_t n = static_cast<size_t>(B) * L * H * d;
  const size_t ns = static_cast<size_t>(B) * H * ((L + 127) / 128) * 4;
  if (overlaps(codes, n, x, 2 * n) || overlaps(scales, ns, x, 2 * n) || overlaps(scales, ns, codes, n))
    return fail(RA_ERR_INVALID_ARG, "outputs overlap the input or each other");
  int sms = 0;
  ra_status st = device_info(&sms);
  if (st != RA_OK) return st;
  cudaError_t e = ra::launch_quantize_fp8(static_cast<const __nv_bfloat16*>(x),
                                          static_cast<uint8_t*>(codes), scales, B, L, H, d,
                                          reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "quantize launch: %s", cudaGetErrorString(e));
  return ok();
}

ra_status ring_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                            const float* sk, const float* sv, void* out, float* lse, int B, int Hq,
                            int Hkv, int64_t L, int d, int n_ring, int causal, float scale,
                            ra_stream_t stream) {
  ra_status st = check_forward_shape(B, Hq, Hkv, L, d, n_ring, causal, scale);
  if (st != RA_OK) return st;
  if (d != 128) return fail(RA_ERR_UNSUPPORTED, "the FP8 forward supports head dim 128 (got %d)", d);
  if ((L / n_ring) % 128 != 0)
    return fail(RA_ERR_UNSUPPORTED, "the FP8 forward needs L / n_ring to be a multiple of 128");
  if (static_cast<long long>(B) * Hq * L == 0) return ok();
  if (!q8 || !k8 || !v8 || !sq || !sk || !sv || !out || !lse)
    return fail(RA_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[8] = {q8, k8, v8, sq, sk, sv, out, lse};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return fail(RA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const long long T = L / 128;
  const size_t nq = static_cast<size_t>(B) * L * Hq * 128;
  const size_t nkv = static_cast<size_t>(B) * L * Hkv * 128;
  const size_t nsq = static_cast<size_t>(B) * Hq * T * 4, nskv = static_cast<size_t>(B) * Hkv * T * 4;
  const size_t no = 2 * nq, nl = static_cast<size_t>(B) * Hq * L * 4;
  const void* ins[6] = {q8, k8, v8, sq, sk, sv};
  const size_t in_n[6] = {nq, nkv, nkv, nsq, nskv, nskv};
  for (int i = 0; i < 6; ++i)
    if (overlaps(out, no, ins[i], in_n[i]) || overlaps(lse, nl, ins[i], in_n[i]))
      return fail(RA_ERR_INVALID_ARG, "outputs overlap the inputs");
  if (overlaps(out, no, lse, nl)) return fail(RA_ERR_INVALID_ARG, "out and lse overlap");

  int sms = 0;
  if ((st = device_info(&sms)) != RA_OK) return st;
  ra::Fp8FwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const long long rows = static_cast<long long>(B) * L;
  if ((st = make_map_e4m3(&prm.tm_q, q8, Hq, rows)) != RA_OK) return st;
  if ((st = make_map_e4m3(&prm.tm_k, k8, Hkv, rows)) != RA_OK) return st;
  if ((st = make_map_e4m3(&prm.tm_v, v8, Hkv, rows)) != RA_OK) return st;
  prm.sq = sq;
  prm.sk = sk;
  prm.sv = sv;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.L = static_cast<int>(L);
  prm.n_ring = n_ring;
  prm.blk_len = static_cast<int>(L / n_ring);
  prm.causal = causal;
  prm.tiles_per_blk = prm.blk_len / 128;
  prm.pair_heads = prm.group >= 2 ? 1 : 0;
  prm.head_slots = (prm.group + 1) / 2;
  prm.pairs_per_blk = (prm.tiles_per_blk + 1) / 2;
  prm.n_tiles = static_cast<int>(T);
  const long long units =
      prm.pair_heads
          ? static_cast<long long>(B) * Hkv * prm.head_slots * n_ring * prm.tiles_per_blk
          : static_cast<long long>(B) * Hq * n_ring * prm.pairs_per_blk;
  if (units >= (1ll << 31)) return fail(RA_ERR_INVALID_ARG, "problem too large (%lld work units)", units);
  prm.total_units = static_cast<int>(units);
  const int sched = g_schedule.load();
  prm.head_major = sched == RA_SCHEDULE_HEAD_MAJOR ||
                   (sched == RA_SCHEDULE_AUTO && 2.0 * static_cast<double>(nkv) > kHeadMajorKvBytes);
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  prm.wait_limit_ns = g_wait_limit_ns.load();
  prm.debug_flags = g_debug_flags.load();
  long long grid = sms;
  const int cap = g_max_ctas.load();
  if (cap > 0 && cap < grid) grid = cap;
  if (grid > prm.total_units) grid = prm.total_units;
  cudaError_t e = ra::next_ticket_counter(reinterpret_cast<cudaStream_t>(stream), &prm.tickets);
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "work queue reset: %s", cudaGetErrorString(e));
  e = ra::launch_fwd_fp8(prm, static_cast<int>(grid), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "FP8 forward launch: %s", cudaGetErrorString(e));
  return ok();
}

ra_status ring_attn_check_status(ra_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  unsigned long long v = 0, vb = 0, v8 = 0;
  e = ra::read_and_clear_status(&v);
  if (e == cudaSuccess) e = ra::read_and_clear_bwd_status(&vb);
  if (e == cudaSuccess) e = ra::read_and_clear_fp8_status(&v8);
  if (e != cudaSuccess) return fail(RA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  if (v == 0) v = vb;
  if (v == 0) v = v8;
  if (v == 0) return ok();
  const unsigned code = static_cast<unsigned>(v >> 32);
  const unsigned site = static_cast<unsigned>((v >> 16) & 0xFFFF);
  const unsigned cta = static_cast<unsigned>(v & 0xFFFF);
  return fail(static_cast<ra_status>(code), "device wait ran out (site %u, CTA %u)", site, cta);
}

ra_status ring_attn_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns == 0 ? 5000000000ull : ns);
  return ok();
}

ra_status ring_attn_set_max_ctas(int n) {
  if (n < 0) return fail(RA_ERR_INVALID_ARG, "max CTAs must be >= 0");
  g_max_ctas.store(n);
  return ok();
}

ra_status ring_attn_set_schedule(int schedule) {
  if (schedule != RA_SCHEDULE_AUTO && schedule != RA_SCHEDULE_LONGEST_FIRST &&
      schedule != RA_SCHEDULE_HEAD_MAJOR)
    return fail(RA_ERR_INVALID_ARG, "unknown schedule %d", schedule);
  g_schedule.store(schedule);
  return ok();
}

ra_status ring_attn_debug_inject(unsigned flags) {
  if (flags & ~1u) return fail(RA_ERR_INVALID_ARG, "unknown debug flag bits 0x%x", flags & ~1u);
  g_debug_flags.store(flags);
  return ok();
}

const char* ring_attn_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "RA_OK";
    case RA_ERR_INVALID_ARG: return "RA_ERR_INVALID_ARG";
    case RA_ERR_UNSUPPORTED: return "RA_ERR_UNSUPPORTED";
    case RA_ERR_CUDA: return "RA_ERR_CUDA";
    case RA_ERR_TIMEOUT: return "RA_ERR_TIMEOUT";
  }
  return "RA_ERR_UNKNOWN";
}

const char* ring_attn_last_error(void) { return g_last_error.c_str(); }

int ring_attn_version(void) { return 104; }

}  // extern "C"
