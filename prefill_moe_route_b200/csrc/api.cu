// api.cu -- the C ABI of libmoe_b200.so (include/moe_b200.h): argument
// checks, device guard, workspace plan, TMA tensor maps, and the launch
// sequence of one MoE call:
//   route+quant (+ sort counts) -> sort scatter -> GEMM1 (+SwiGLU, mid quant)
//   -> GEMM2 -> combine,
// chained with programmatic dependent launch so each kernel's prologue
// overlaps the previous kernel's tail.  Nothing here synchronizes the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "internal.h"

namespace moe {

cudaError_t launch_route(const RouteParams& p, cudaStream_t st);
cudaError_t launch_align(const RouteParams& p, cudaStream_t st);
cudaError_t launch_pack_bsf(const RouteParams& p, int num_sms, cudaStream_t st);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t st);
cudaError_t launch_round_bf16(const float* in, uint16_t* out, int64_t n, cudaStream_t st);
cudaError_t run_tensor_probe(int kind, int iters, cudaStream_t st, double* tflops, double* mac_per_clk);
cudaError_t launch_quant_mxfp4(const float* w, int64_t nblocks, uint8_t* q, uint8_t* s, cudaStream_t st);
cudaError_t launch_pack_mx_scales(const uint8_t* s, int64_t batch, int rows, int K, uint8_t* out, cudaStream_t st);
cudaError_t launch_quant_fp8(const float* w, int64_t batch, int rows, int K, uint8_t* q, float* s,
                             cudaStream_t st);
cudaError_t launch_gemm1(int wfmt, int nt, const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p,
                         int grid, cudaStream_t st);
cudaError_t launch_gemm2(int wfmt, int nt, const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p,
                         int grid, cudaStream_t st);
int small_max_clusters(int dev);
int small_cluster_size();
cudaError_t launch_small(const CUtensorMap& w13, const CUtensorMap& w2, const CUtensorMap& mid,
                         const SmallParams& p, int nclusters, cudaStream_t st);

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Text of the last failure on this thread (moe_last_error).
static thread_local char g_last_error[256] = "";

static int fail(int code, const char* what, cudaError_t e = cudaSuccess) {
  if (e != cudaSuccess)
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
  else
    std::snprintf(g_last_error, sizeof(g_last_error), "%s", what);
  return code;
}

int make_plan(const moe_shape_t& s, int num_sms, Plan* p) {
  if (s.M < 1 || s.E < 1 || s.topk < 1 || s.H < 128 || s.I < 128) return MOE_ERR_INVALID_ARG;
  if (s.wfmt != MOE_W_MXFP4 && s.wfmt != MOE_W_FP8_BLOCK128) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(s.routed_scale)) return MOE_ERR_INVALID_ARG;
  if (s.E > kMaxE || s.topk > kMaxTopk || s.topk > s.E) return MOE_ERR_UNSUPPORTED;
  if (s.I % 128 != 0 || s.H % (s.wfmt == MOE_W_MXFP4 ? 256 : 128) != 0) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)s.M * s.topk > (1 << 20) || s.H > 65536 || s.I > 65536) return MOE_ERR_UNSUPPORTED;
  std::memset(p, 0, sizeof(*p));
  p->M = s.M; p->H = s.H; p->I = s.I; p->E = s.E; p->topk = s.topk; p->wfmt = s.wfmt;
  p->routed_scale = s.routed_scale;
  p->P = s.M * s.topk;
  // one tile per expert whenever every token fits: a token picks an expert once.
  // Block-FP8 with 32 or more pairs per expert on average takes 128-pair tiles
  // (the wide kernels: pairs on the MMA's M side, 256 weight rows on N).
  // Measured on B200 (H = 6144, E = 256, top-8, I = 512, Zipf routing), whole
  // call wide / narrow: M = 512 (16 pairs per expert) 574 / 532 us, M = 1024
  // 608 / 625, M = 2048 734 / 853, M = 4096 1030 / 1333.
  int nt = s.M <= 16 ? 16 : (s.M <= 32 ? 32 : 64);
  if (s.wfmt == MOE_W_FP8_BLOCK128 && s.M > 64 && (int64_t)s.M * s.topk >= 32 * (int64_t)s.E) nt = 128;
  p->nt1 = nt;
  p->nt2 = nt;
  p->kst1 = s.wfmt == MOE_W_MXFP4 ? s.H / 256 : s.H / 128;
  p->kst2 = s.I / 128;
  p->j1 = s.I / 128;
  p->ht2 = s.H / 128;
  // K splits for GEMM1 when few (expert, n-tile) groups would leave SMs idle
  p->split1 = 1;
  if (s.wfmt == MOE_W_MXFP4 && p->P <= 512) {
    const double distinct = s.E * (1.0 - std::pow(1.0 - (double)s.topk / s.E, (double)s.M));
    const int est = std::max(1, (int)std::ceil(distinct)) * p->j1;
    for (int d = 1; d <= p->kst1; ++d)
      if (p->kst1 % d == 0 && p->kst1 / d >= 2 && d <= 8 && est * d <= 2 * num_sms) p->split1 = d;
  }
  p->groups1 = (std::min(s.E, p->P) + p->P / nt + 1) * p->j1;

  const size_t P = p->P, M = s.M, H = s.H, I = s.I, E = s.E;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes, 256); return r; };
  p->o_status = take(16);
  p->o_ids = take(P * 4);
  p->o_w = take(P * 4);
  p->o_counts = take(E * 4);
  p->o_offsets = take((E + 1) * 4);
  p->o_sorted = take(P * 4);
  p->o_inv = take(P * 4);
  p->o_tiles1 = take((E + 1) * 4);
  p->o_tiles2 = take((E + 1) * 4);
  if (s.wfmt == MOE_W_MXFP4) { p->o_xq = take(M * H / 2); p->o_xs = take(M * H / 32); }
  else { p->o_xq = take(M * H); p->o_xs = take(M * (H / 128) * 4); }
  p->o_midq = take(P * I);
  p->o_midqs = take(P * (I / 128) * 4);
  p->o_y = take(P * H * 2);
  p->o_cnt1 = take((size_t)p->groups1 * 4);
  p->o_sync = take(16);
  p->o_flags = take(E * 16 * 4);
  // Decode-sized MXFP4 calls run as one launch (small.cu) while M * topk <= 64:
  // measured on B200 (H = 6144, E = 256, top-8), the single kernel is faster up
  // to M = 8 and the grouped kernels from M = 12 on spread routing (and at M =
  // 16, I = 512 on skewed routing); the kernel itself takes M <= 16, M * topk <=
  // 256.  MOE_FORCE_PATH=large keeps every call on the grouped kernels,
  // MOE_FORCE_PATH=small takes the single kernel wherever it can run.
  static const int force = [] {
    const char* e = std::getenv("MOE_FORCE_PATH");
    return !e ? 0 : std::strcmp(e, "large") == 0 ? 1 : std::strcmp(e, "small") == 0 ? 2 : 0;
  }();
  const bool small_fits = s.wfmt == MOE_W_MXFP4 && s.M <= 16 && p->P <= 256 && s.I <= 1024 && s.H <= 8192;
  p->small = small_fits && (force == 2 || (force == 0 && p->P <= 64));
  p->o_midsf = take(p->small ? E * (I / 128) * 256 : 0);
  p->o_midt = take(p->small ? E * 16 * I : 0);
  p->o_xpart = take(p->small ? (H / 128) * 128 * 16 * 4 : 0);
  p->o_xflag = take(p->small ? (H / 128) * 4 : 0);
  p->o_part = take(p->split1 > 1 ? (size_t)p->groups1 * p->split1 * nt * 256 * 4 : 0);
  // the sort's chunks: about 512 pairs each, one scatter CTA per chunk
  p->chunk_tokens = std::max(1, 512 / s.topk);
  p->nchunks = (s.M + p->chunk_tokens - 1) / p->chunk_tokens;
  p->o_chunk = take((size_t)p->nchunks * E * 4);
  p->o_sortw = take(P * 4);
  // packed operand scales, one 512-byte block per (token tile, 128-column chunk);
  // GEMM2's tiles are GEMM1's (nt2 == nt1), so GEMM1's epilogue can fill them
  p->tiles_max = (int)std::min(E, P) + (int)(P / nt) + 1;
  p->o_bsf1 = take((size_t)p->tiles_max * (H / 128) * 512);
  p->o_bsf2 = take((size_t)p->tiles_max * (I / 128) * 512);
  p->o_xg = take(P * (s.wfmt == MOE_W_MXFP4 ? H / 2 : H));
  p->total = o;
  return MOE_OK;
}

// ---------------------------------------------------------------- helpers
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bd[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bd[i] = box[i]; }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, dt, rank, const_cast<void*>(base), gd, gs, bd, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int sm_count(int dev) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static uint64_t wait_timeout_ns() {
  static uint64_t v = [] {
    const char* e = std::getenv("MOE_WAIT_TIMEOUT_MS");
    long ms = e ? std::atol(e) : 2000;
    if (ms <= 0) ms = 2000;
    return (uint64_t)ms * 1000000ull;
  }();
  return v;
}

// Test knob MOE_TEST_WITHHOLD_FLAG=n: the first n single-launch calls of the
// process leave one mid flag unpublished, so that the device-side waits on it
// run out (bounded by MOE_WAIT_TIMEOUT_MS) and the call reports
// MOE_ERR_DEVICE_TIMEOUT through the status word.  Read once per process.
static std::atomic<int> g_withhold_left{-1};
static int take_withhold() {
  int left = g_withhold_left.load();
  if (left < 0) {
    const char* e = std::getenv("MOE_TEST_WITHHOLD_FLAG");
    int v = e ? std::atoi(e) : 0;
    int expect = -1;
    g_withhold_left.compare_exchange_strong(expect, v < 0 ? 0 : v);
  }
  left = g_withhold_left.load();
  while (left > 0 && !g_withhold_left.compare_exchange_weak(left, left - 1)) {}
  return left > 0 ? 1 : 0;
}

// Device of a device pointer, -1 if it is not device memory.
static int device_of(const void* ptr) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) { cudaGetLastError(); return -1; }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return -1;
  return a.device;
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// Device of the stream, checked against every pointer; <0 is an error code.
// Pointer attributes are not queried while the stream is being captured into
// a CUDA graph (the eager calls before capture check the same buffers).
static int resolve_device(void* stream, const void* const* ptrs, int n) {
  int dev = -1;
  cudaError_t e;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (stream && (e = cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "cudaStreamIsCapturing", e);
  if (stream && cap == cudaStreamCaptureStatusNone) {
    if ((e = cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &dev)) != cudaSuccess) {
      cudaGetLastError();
      return fail(MOE_ERR_CUDA, "cudaStreamGetDevice", e);
    }
  } else if ((e = cudaGetDevice(&dev)) != cudaSuccess) {
    // a capturing stream cannot be asked for its device: the caller's
    // current device is the one being captured
    return fail(MOE_ERR_CUDA, "cudaGetDevice", e);
  }
  if (cap != cudaStreamCaptureStatusNone) return dev;
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) continue;
    const int d = device_of(ptrs[i]);
    if (d < 0) return fail(MOE_ERR_INVALID_ARG, "a tensor argument is not device memory");
    if (d != dev) return fail(MOE_ERR_DEVICE_MISMATCH, "a tensor argument lives on another device than the stream");
  }
  return dev;
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Scratch of moe_forward_static, for callers that cannot allocate device
// memory: one fixed array per device that loads the library, held until the
// process exits.  Host code only ever uses its device address, looked up once
// per device with that device current (cudaGetSymbolAddress): the symbol's
// host-side name is not a device address.
static __device__ __align__(256) uint8_t g_static_scratch[MOE_STATIC_SCRATCH_BYTES];
static void* g_static_scratch_addr[64] = {nullptr};
static std::mutex g_static_scratch_mu;

static int static_scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "moe_forward_static: device index above 63");
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);   // the device is current here
    if (e != cudaSuccess || !p) return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress of the static scratch", e);
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_last_error(void) { return g_last_error; }

int moe_workspace_size(const moe_shape_t* shape, size_t* bytes) {
  if (!shape || !bytes) return MOE_ERR_INVALID_ARG;
  Plan p;
  int rc = make_plan(*shape, 148, &p);
  if (rc != MOE_OK) return rc;
  // the split-K plan depends on the SM count; size for the largest split
  Plan q;
  make_plan(*shape, 1 << 20, &q);
  *bytes = std::max(p.total, q.total);
  return MOE_OK;
}

int moe_workspace_layout(const moe_shape_t* shape, moe_ws_layout_t* l) {
  if (!shape || !l) return MOE_ERR_INVALID_ARG;
  Plan p;
  int rc = make_plan(*shape, 148, &p);
  if (rc != MOE_OK) return rc;
  size_t total = 0;
  moe_workspace_size(shape, &total);
  l->status = p.o_status; l->topk_ids = p.o_ids; l->topk_w = p.o_w; l->counts = p.o_counts;
  l->offsets = p.o_offsets; l->sorted_pairs = p.o_sorted; l->inv = p.o_inv;
  l->midq = p.o_midq; l->midqs = p.o_midqs; l->total_bytes = total;
  return MOE_OK;
}

int moe_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  const void* ptrs[1] = {workspace};
  int dev = resolve_device(stream, ptrs, 1);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  if (cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_route(const moe_shape_t* shape, const float* logits, const float* bias, int32_t* topk_ids,
              float* topk_w, void* stream) {
  if (!shape || !logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  Plan pl;
  int rc = make_plan(*shape, 148, &pl);
  if (rc != MOE_OK) return rc;
  const void* ptrs[4] = {logits, bias, topk_ids, topk_w};
  int dev = resolve_device(stream, ptrs, 4);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  RouteParams r = {};
  r.logits = logits; r.bias = bias; r.x = nullptr;
  r.topk_ids = topk_ids; r.topk_w = topk_w;
  r.M = shape->M; r.E = shape->E; r.topk = shape->topk; r.H = shape->H; r.wfmt = shape->wfmt;
  r.routed_scale = shape->routed_scale; r.nt1 = pl.nt1; r.nt2 = pl.nt2; r.do_align = 0;
  return launch_route(r, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// logits (+ bias) route inside the call; ids_in / w_in (both set, logits
// ignored) take the caller's selection.
static int forward_impl(const moe_shape_t* shape, const void* x, const float* logits, const float* bias,
                        const int32_t* ids_in, const float* w_in,
                        const void* w13, const void* w13_scales, const void* w2, const void* w2_scales, void* out,
                        void* workspace, size_t ws_bytes, void* stream, void* const* events,
                        bool out_f32 = false) {
  const bool routed = ids_in != nullptr;
  if (!shape || !x || !w13 || !w13_scales || !w2 || !w2_scales || !out || !workspace ||
      (routed ? !w_in : !logits))
    return fail(MOE_ERR_INVALID_ARG, "moe_forward: null pointer argument");
  if (routed) { logits = nullptr; bias = nullptr; }
  const void* ptrs[11] = {x, logits, bias, w13, w13_scales, w2, w2_scales, out, workspace, ids_in, w_in};
  for (int i = 0; i < 11; ++i)
    if (ptrs[i] && !aligned(ptrs[i], 16)) return fail(MOE_ERR_INVALID_ARG, "moe_forward: pointer not 16-byte aligned");
  if (!aligned(w13, 32) || !aligned(w2, 32) || !aligned(workspace, 256))
    return fail(MOE_ERR_INVALID_ARG, "moe_forward: w13/w2 need 32-byte, workspace 256-byte alignment");
  if (out == x || (logits && out == logits) || out == workspace || (routed && (out == ids_in || out == w_in)))
    return fail(MOE_ERR_INVALID_ARG, "moe_forward: out aliases an input");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool mx = shape->wfmt == MOE_W_MXFP4;

  // A call with the same shape and buffers as this thread's previous call
  // reuses its device check and tensor maps (host cost of a repeated call).
  struct CallCache {
    bool valid = false;
    moe_shape_t shape;
    const void* ptrs[11];
    size_t ws_bytes;
    int dev;
    Plan pl;
    CUtensorMap mA1, mB1, mA2, mB2;
  };
  static thread_local CallCache cache;
  int dev = -1;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (stream && cudaStreamIsCapturing(st, &cap) != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaStreamIsCapturing");
  if (stream && cap == cudaStreamCaptureStatusNone) {
    cudaError_t e = cudaStreamGetDevice(st, &dev);
    if (e != cudaSuccess) { cudaGetLastError(); return fail(MOE_ERR_CUDA, "cudaStreamGetDevice", e); }
  } else if (cudaGetDevice(&dev) != cudaSuccess) {
    return fail(MOE_ERR_CUDA, "cudaGetDevice");
  }
  const bool hit = cache.valid && cache.dev == dev && cache.ws_bytes == ws_bytes &&
                   std::memcmp(&cache.shape, shape, sizeof(moe_shape_t)) == 0 &&
                   std::memcmp(cache.ptrs, ptrs, sizeof(ptrs)) == 0;
  if (!hit) {
    cache.valid = false;
    const int d = resolve_device(stream, ptrs, 11);
    if (d < 0) return d;
    dev = d;
  }
  DeviceGuard g(dev);
  const int sms = sm_count(dev);
  Plan pl;
  if (hit) {
    pl = cache.pl;
  } else {
    int rc = make_plan(*shape, sms, &pl);
    if (rc != MOE_OK) return fail(rc, "moe_forward: unsupported shape");
    // the single kernel needs its clusters co-resident and at most 2 h-tiles per cluster
    if (pl.small) {
      const int ncl = std::min(small_max_clusters(dev), sms / small_cluster_size());
      if (ncl <= 0 || pl.H / 128 > 2 * ncl) pl.small = false;
    }
  }
  if (ws_bytes < pl.total) return fail(MOE_ERR_WORKSPACE, "moe_forward: workspace smaller than moe_workspace_size");
  const uint64_t M = pl.M, H = pl.H, I = pl.I, E = pl.E, P = pl.P;

  // ---- tensor maps
  CUtensorMap mA1, mB1, mA2, mB2;
  if (hit) {
    mA1 = cache.mA1; mB1 = cache.mB1; mA2 = cache.mA2; mB2 = cache.mB2;
  } else {
    bool ok = true;
    {
      const uint64_t kb = mx ? H / 2 : H;
      uint64_t d[3] = {kb, 2 * I, E}, s[2] = {kb, 2 * I * kb};
      uint32_t b[3] = {128, 128, 1};
      ok &= make_map(&mA1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w13, d, s, b);
      // the token rows in sorted-pair order: one tile of nt1 rows per stage
      uint64_t d2[2] = {kb, P}, s2[1] = {kb};
      uint32_t b2[2] = {128, (uint32_t)pl.nt1};
      ok &= make_map(&mB1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, ws + pl.o_xg, d2, s2, b2);
    }
    {
      const uint64_t rowb = mx ? I / 2 : I;
      uint64_t d[3] = {I, H, E}, s[2] = {rowb, H * rowb};
      uint32_t b[3] = {128, 128, 1};
      ok &= make_map(&mA2, mx ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w2, d, s,
                     b);
      // mid as GEMM2's B operand: sorted pairs (grouped kernels) or, for the
      // single-launch kernel, 16 token rows per expert
      uint64_t d2[2] = {I, pl.small ? (uint64_t)E * 16 : P}, s2[1] = {I};
      uint32_t b2[2] = {128, (uint32_t)pl.nt2};
      ok &= make_map(&mB2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, ws + (pl.small ? pl.o_midt : pl.o_midq), d2, s2, b2);
    }
    if (!ok) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled rejected a tensor map");
    cache.shape = *shape;
    std::memcpy(cache.ptrs, ptrs, sizeof(ptrs));
    cache.ws_bytes = ws_bytes;
    cache.dev = dev;
    cache.pl = pl;
    cache.mA1 = mA1; cache.mB1 = mB1; cache.mA2 = mA2; cache.mB2 = mB2;
    cache.valid = true;
  }

  int32_t* status = reinterpret_cast<int32_t*>(ws + pl.o_status);
  // inside a graph capture an event must be an external record node to keep its timestamp
  auto mark = [&](int i) {
    if (!events) return true;
    const unsigned flags = cap != cudaStreamCaptureStatusNone ? cudaEventRecordExternal : cudaEventRecordDefault;
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), st, flags) == cudaSuccess;
  };
  cudaError_t le;

  const int ncl = pl.small ? small_max_clusters(dev) : 0;
  if (pl.small && ncl > 0) {
    // ---- the whole call in one launch
    SmallParams sp = {};
    sp.x = static_cast<const uint16_t*>(x); sp.logits = logits; sp.bias = bias;
    sp.ids_in = ids_in; sp.w_in = w_in;
    sp.w2 = static_cast<const uint8_t*>(w2);
    sp.s13 = static_cast<const uint8_t*>(w13_scales); sp.s2 = static_cast<const uint8_t*>(w2_scales);
    sp.out = static_cast<uint16_t*>(out); sp.status = status;
    sp.out_f32 = out_f32 ? static_cast<float*>(out) : nullptr;
    sp.sync = reinterpret_cast<int32_t*>(ws + pl.o_sync);
    sp.flags = reinterpret_cast<int32_t*>(ws + pl.o_flags);
    sp.topk_ids = reinterpret_cast<int32_t*>(ws + pl.o_ids);
    sp.topk_w = reinterpret_cast<float*>(ws + pl.o_w);
    sp.counts = reinterpret_cast<int32_t*>(ws + pl.o_counts);
    sp.offsets = reinterpret_cast<int32_t*>(ws + pl.o_offsets);
    sp.sorted_pairs = reinterpret_cast<int32_t*>(ws + pl.o_sorted);
    sp.inv = reinterpret_cast<int32_t*>(ws + pl.o_inv);
    sp.midq = ws + pl.o_midq; sp.midqs = reinterpret_cast<float*>(ws + pl.o_midqs);
    sp.midsf = reinterpret_cast<uint32_t*>(ws + pl.o_midsf);
    sp.midt = ws + pl.o_midt;
    sp.xpart = reinterpret_cast<float*>(ws + pl.o_xpart);
    sp.xflag = reinterpret_cast<int32_t*>(ws + pl.o_xflag);
    sp.M = pl.M; sp.H = pl.H; sp.I = pl.I; sp.E = pl.E; sp.topk = pl.topk;
    sp.routed_scale = pl.routed_scale; sp.timeout_ns = wait_timeout_ns();
    sp.test_withhold = take_withhold();
    if (!mark(0)) return fail(MOE_ERR_CUDA, "cudaEventRecord");
    if ((le = launch_small(mA1, mA2, mB2, sp, std::min(ncl, sms / small_cluster_size()), st)) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "single-launch kernel", le);
    for (int i = 1; i < 5; ++i)
      if (!mark(i)) return fail(MOE_ERR_CUDA, "cudaEventRecord");
    return MOE_OK;
  }

  // ---- 1. route + activation quant + align
  RouteParams r = {};
  r.logits = logits; r.bias = bias; r.x = static_cast<const uint16_t*>(x);
  r.ids_in = ids_in; r.w_in = w_in;
  r.topk_ids = reinterpret_cast<int32_t*>(ws + pl.o_ids);
  r.topk_w = reinterpret_cast<float*>(ws + pl.o_w);
  r.xq = ws + pl.o_xq; r.xs = ws + pl.o_xs; r.status = status;
  r.counts = reinterpret_cast<int32_t*>(ws + pl.o_counts);
  r.offsets = reinterpret_cast<int32_t*>(ws + pl.o_offsets);
  r.sorted_pairs = reinterpret_cast<int32_t*>(ws + pl.o_sorted);
  r.inv = reinterpret_cast<int32_t*>(ws + pl.o_inv);
  r.sorted_w = reinterpret_cast<float*>(ws + pl.o_sortw);
  r.bsf = reinterpret_cast<uint32_t*>(ws + pl.o_bsf1);
  r.xg = ws + pl.o_xg;
  r.tiles1 = reinterpret_cast<int32_t*>(ws + pl.o_tiles1);
  r.tiles2 = reinterpret_cast<int32_t*>(ws + pl.o_tiles2);
  r.M = pl.M; r.E = pl.E; r.topk = pl.topk; r.H = pl.H; r.wfmt = pl.wfmt;
  r.nt1 = pl.nt1; r.nt2 = pl.nt2; r.routed_scale = pl.routed_scale; r.do_align = 1;
  r.chunk_cnt = reinterpret_cast<int32_t*>(ws + pl.o_chunk);
  r.chunk_tokens = pl.chunk_tokens; r.chunk_pairs = pl.chunk_tokens * pl.topk; r.nchunks = pl.nchunks;
  if (!mark(0)) return fail(MOE_ERR_CUDA, "cudaEventRecord");
  if ((le = launch_route(r, st)) != cudaSuccess) return fail(MOE_ERR_CUDA, "route kernel launch", le);
  if ((le = launch_align(r, st)) != cudaSuccess) return fail(MOE_ERR_CUDA, "align kernel launch", le);
  if ((le = launch_pack_bsf(r, sms, st)) != cudaSuccess) return fail(MOE_ERR_CUDA, "scale packing kernel launch", le);
  if (!mark(1)) return fail(MOE_ERR_CUDA, "cudaEventRecord");

  // ---- 2. GEMM1 + SwiGLU + mid quantization
  GemmParams g1 = {};
  g1.offsets = r.offsets; g1.counts = r.counts; g1.sorted_pairs = r.sorted_pairs; g1.tiles = r.tiles1;
  if (mx) g1.sfa_u8 = static_cast<const uint8_t*>(w13_scales);
  else g1.sfa_f32 = static_cast<const float*>(w13_scales);
  g1.bsf = ws + pl.o_bsf1; g1.nchb = pl.H / 128;
  g1.bsf_out = reinterpret_cast<uint32_t*>(ws + pl.o_bsf2);
  g1.midq = ws + pl.o_midq; g1.midqs = reinterpret_cast<float*>(ws + pl.o_midqs);
  g1.part = reinterpret_cast<float*>(ws + pl.o_part); g1.cnt = reinterpret_cast<int32_t*>(ws + pl.o_cnt1);
  g1.status = status;
  g1.M = pl.M; g1.H = pl.H; g1.I = pl.I; g1.E = pl.E; g1.topk = pl.topk; g1.P = pl.P;
  g1.kst = pl.kst1; g1.split = pl.split1; g1.jn = pl.j1; g1.timeout_ns = wait_timeout_ns();
  const int bound1 = (std::min(pl.E, pl.P) + pl.P / pl.nt1 + 1) * pl.j1 * pl.split1;
  if ((le = launch_gemm1(pl.wfmt, pl.nt1, mA1, mB1, g1, std::min(sms, bound1), st)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "GEMM1 kernel launch", le);
  if (!mark(2)) return fail(MOE_ERR_CUDA, "cudaEventRecord");

  // ---- 3. GEMM2
  GemmParams g2 = g1;
  g2.tiles = r.tiles2;
  if (mx) { g2.sfa_u8 = static_cast<const uint8_t*>(w2_scales); g2.sfa_f32 = nullptr; }
  else { g2.sfa_f32 = static_cast<const float*>(w2_scales); g2.sfa_u8 = nullptr; }
  g2.bsf = ws + pl.o_bsf2; g2.nchb = pl.I / 128; g2.bsf_out = nullptr;
  g2.yw = reinterpret_cast<uint16_t*>(ws + pl.o_y);
  g2.sorted_w = r.sorted_w;
  g2.kst = pl.kst2; g2.split = 1; g2.jn = (pl.ht2 + 1) / 2;   // a GEMM2 task covers two 128-row h-tiles
  const int bound2 = (std::min(pl.E, pl.P) + pl.P / pl.nt2 + 1) * g2.jn;
  if ((le = launch_gemm2(pl.wfmt, pl.nt2, mA2, mB2, g2, std::min(sms, bound2), st)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "GEMM2 kernel launch", le);
  if (!mark(3)) return fail(MOE_ERR_CUDA, "cudaEventRecord");

  // ---- 4. combine
  CombineParams c = {};
  c.yw = g2.yw; c.inv = r.inv; c.out = static_cast<uint16_t*>(out);
  c.out_f32 = out_f32 ? static_cast<float*>(out) : nullptr;
  c.M = pl.M; c.H = pl.H; c.topk = pl.topk;
  if ((le = launch_combine(c, st)) != cudaSuccess) return fail(MOE_ERR_CUDA, "combine kernel launch", le);
  if (!mark(4)) return fail(MOE_ERR_CUDA, "cudaEventRecord");
  return MOE_OK;
}

int moe_forward(const moe_shape_t* shape, const void* x, const float* logits, const float* bias,
                const void* w13, const void* w13_scales, const void* w2, const void* w2_scales, void* out,
                void* workspace, size_t ws_bytes, void* stream) {
  return forward_impl(shape, x, logits, bias, nullptr, nullptr, w13, w13_scales, w2, w2_scales, out, workspace,
                      ws_bytes, stream, nullptr);
}

int moe_forward_partial(const moe_shape_t* shape, const void* x, const float* logits, const float* bias,
                        const void* w13, const void* w13_scales, const void* w2, const void* w2_scales,
                        float* out_partial, void* workspace, size_t ws_bytes, void* stream) {
  if (!out_partial) return fail(MOE_ERR_INVALID_ARG, "moe_forward_partial: null pointer argument");
  return forward_impl(shape, x, logits, bias, nullptr, nullptr, w13, w13_scales, w2, w2_scales, out_partial,
                      workspace, ws_bytes, stream, nullptr, true);
}

int moe_round_bf16(const float* in, void* out, int64_t n, void* stream) {
  if (!in || !out || n < 0 || n % 8) return fail(MOE_ERR_INVALID_ARG, "moe_round_bf16: null pointer or n not a multiple of 8");
  if (!aligned(in, 16) || !aligned(out, 16)) return fail(MOE_ERR_INVALID_ARG, "moe_round_bf16: misaligned pointer");
  if (n == 0) return MOE_OK;
  const void* ptrs[2] = {in, out};
  const int dev = resolve_device(stream, ptrs, 2);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  const cudaError_t e = launch_round_bf16(in, static_cast<uint16_t*>(out), n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : fail(MOE_ERR_CUDA, "moe_round_bf16", e);
}

int moe_probe_tensor_peak(int kind, int iters, double* tflops, double* mac_per_clk, void* stream) {
  if (kind < MOE_PROBE_FP8 || kind > MOE_PROBE_BF16 || iters < 1 || iters > 100000 || !tflops || !mac_per_clk)
    return fail(MOE_ERR_INVALID_ARG, "moe_probe_tensor_peak: bad kind or count, or a null output");
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e;
  if (stream && (e = cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "cudaStreamIsCapturing", e);
  if (cap != cudaStreamCaptureStatusNone)
    return fail(MOE_ERR_INVALID_ARG, "moe_probe_tensor_peak: the stream is being captured");
  const int dev = resolve_device(stream, nullptr, 0);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  double tf = 0.0, mpc = 0.0;
  if ((e = run_tensor_probe(kind, iters, static_cast<cudaStream_t>(stream), &tf, &mpc)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "moe_probe_tensor_peak", e);
  if (!(tf > 0.0)) return fail(MOE_ERR_DEVICE_TIMEOUT, "moe_probe_tensor_peak: an SM's MMAs did not complete in time");
  *tflops = tf;
  *mac_per_clk = mpc;
  return MOE_OK;
}

int moe_forward_routed(const moe_shape_t* shape, const void* x, const int32_t* topk_ids, const float* topk_w,
                       const void* w13, const void* w13_scales, const void* w2, const void* w2_scales, void* out,
                       void* workspace, size_t ws_bytes, void* stream) {
  if (!topk_ids || !topk_w) return fail(MOE_ERR_INVALID_ARG, "moe_forward_routed: null pointer argument");
  return forward_impl(shape, x, nullptr, nullptr, topk_ids, topk_w, w13, w13_scales, w2, w2_scales, out, workspace,
                      ws_bytes, stream, nullptr);
}

int moe_forward_timed(const moe_shape_t* shape, const void* x, const float* logits, const float* bias,
                      const void* w13, const void* w13_scales, const void* w2, const void* w2_scales, void* out,
                      void* workspace, size_t ws_bytes, void* stream, void* const* events) {
  if (!events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 5; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  return forward_impl(shape, x, logits, bias, nullptr, nullptr, w13, w13_scales, w2, w2_scales, out, workspace,
                      ws_bytes, stream, events);
}

int moe_forward_static(const moe_shape_t* shape, const void* x, const float* logits, const float* bias,
                       const void* w13, const void* w13_scales, const void* w2, const void* w2_scales, void* out,
                       void* stream) {
  if (!shape || !x || !logits || !w13 || !w13_scales || !w2 || !w2_scales || !out)
    return fail(MOE_ERR_INVALID_ARG, "moe_forward_static: null pointer argument");
  const void* ptrs[8] = {x, logits, bias, w13, w13_scales, w2, w2_scales, out};
  const int dev = resolve_device(stream, ptrs, 8);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  Plan pl;
  int rc = make_plan(*shape, sm_count(dev), &pl);
  if (rc != MOE_OK) return fail(rc, "moe_forward_static: unsupported shape");
  if (pl.total > MOE_STATIC_SCRATCH_BYTES) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "moe_forward_static: this shape needs %zu bytes of scratch, more than the %u-byte static "
                  "buffer; use moe_forward with a caller-owned workspace",
                  pl.total, (unsigned)MOE_STATIC_SCRATCH_BYTES);
    return MOE_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if ((rc = static_scratch_address(dev, &scratch)) != MOE_OK) return rc;
  // the shared scratch keeps the previous call's contents: clear the status
  // words, the split-K arrival counters, the call epoch and the flags tagged
  // with it (mid, split h-tile halves) and the sort's chunk counts, which
  // must start at zero
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  cudaError_t e;
  if ((e = cudaMemsetAsync(ws + pl.o_status, 0, 16, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(ws + pl.o_cnt1, 0, (size_t)pl.groups1 * 4, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(ws + pl.o_sync, 0, 16, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(ws + pl.o_flags, 0, (size_t)pl.E * 16 * 4, st)) != cudaSuccess ||
      (pl.small && (e = cudaMemsetAsync(ws + pl.o_xflag, 0, (size_t)(pl.H / 128) * 4, st)) != cudaSuccess) ||
      (e = cudaMemsetAsync(ws + pl.o_chunk, 0, (size_t)pl.nchunks * pl.E * 4, st)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "moe_forward_static: clearing the static scratch", e);
  return forward_impl(shape, x, logits, bias, nullptr, nullptr, w13, w13_scales, w2, w2_scales, out, scratch,
                      MOE_STATIC_SCRATCH_BYTES, stream, nullptr);
}

static int read_and_clear_status(void* ws, cudaStream_t st, int32_t* device_status);

int moe_get_status_static(void* stream, int32_t* device_status) {
  if (!device_status) return fail(MOE_ERR_INVALID_ARG, "moe_get_status_static: null pointer argument");
  const int dev = resolve_device(stream, nullptr, 0);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  void* scratch = nullptr;
  int rc = static_scratch_address(dev, &scratch);
  if (rc != MOE_OK) return rc;
  // the status words sit at the start of every layout (offset 0 of the scratch)
  return read_and_clear_status(scratch, static_cast<cudaStream_t>(stream), device_status);
}

int moe_launches_per_call(const moe_shape_t* shape, int device, int* launches) {
  if (!shape || !launches) return fail(MOE_ERR_INVALID_ARG, "moe_launches_per_call: null pointer argument");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
    return fail(MOE_ERR_INVALID_ARG, "moe_launches_per_call: no such device");
  DeviceGuard g(device);
  Plan pl;
  const int rc = make_plan(*shape, sm_count(device), &pl);
  if (rc != MOE_OK) return fail(rc, "moe_launches_per_call: unsupported shape");
  const int ncl = pl.small ? std::min(small_max_clusters(device), sm_count(device) / small_cluster_size()) : 0;
  *launches = (pl.small && ncl > 0 && pl.H / 128 <= 2 * ncl) ? 1 : 6;
  return MOE_OK;
}

// Reads the status word of the workspace (or static scratch) at `ws` on
// `st`, clears it and the recorded wait site, and maps it to a return code.
static int read_and_clear_status(void* ws, cudaStream_t st, int32_t* device_status) {
  int32_t v = 0;
  cudaError_t e;
  if ((e = cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaStreamSynchronize(st)) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "reading the device status word", e);
  *device_status = v;
  if (v != 0) {
    // clear the status word and the recorded wait site; [1] is the route
    // kernel's arrival counter, already back at zero
    if ((e = cudaMemsetAsync(ws, 0, 4, st)) != cudaSuccess ||
        (e = cudaMemsetAsync(static_cast<uint8_t*>(ws) + 8, 0, 4, st)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "clearing the device status word", e);
    if (v & ST_BAD_INPUT) return MOE_ERR_INVALID_ARG;   // a caller-routed expert ID out of range
    return MOE_ERR_DEVICE_TIMEOUT;
  }
  return MOE_OK;
}

int moe_get_status(void* workspace, void* stream, int32_t* device_status) {
  if (!workspace || !device_status) return MOE_ERR_INVALID_ARG;
  const void* ptrs[1] = {workspace};
  int dev = resolve_device(stream, ptrs, 1);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  return read_and_clear_status(workspace, static_cast<cudaStream_t>(stream), device_status);
}

int moe_quantize_mxfp4(const float* w, int64_t rows, int32_t K, uint8_t* q, uint8_t* scales, void* stream) {
  if (!w || !q || !scales || rows < 1 || K < 32 || K % 32) return MOE_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 16)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[3] = {w, q, scales};
  int dev = resolve_device(stream, ptrs, 3);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  return launch_quant_mxfp4(w, rows * (K / 32), q, scales, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK : MOE_ERR_CUDA;
}

int moe_pack_mxfp4_scales(const uint8_t* scales, int64_t batch, int32_t rows, int32_t K, uint8_t* packed,
                          void* stream) {
  if (!scales || !packed || batch < 1 || rows < 128 || K < 128 || rows % 128 || K % 128)
    return fail(MOE_ERR_INVALID_ARG, "moe_pack_mxfp4_scales: null pointer or rows, K not multiples of 128");
  if (!aligned(scales, 4) || !aligned(packed, 16))
    return fail(MOE_ERR_INVALID_ARG, "moe_pack_mxfp4_scales: misaligned pointer");
  const uint64_t bytes = (uint64_t)batch * rows * (K / 32);
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(scales), b0 = reinterpret_cast<uintptr_t>(packed);
  if (a0 < b0 + bytes && b0 < a0 + bytes) return fail(MOE_ERR_INVALID_ARG, "moe_pack_mxfp4_scales: buffers overlap");
  const void* ptrs[2] = {scales, packed};
  int dev = resolve_device(stream, ptrs, 2);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  const cudaError_t e = launch_pack_mx_scales(scales, batch, rows, K, packed, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : fail(MOE_ERR_CUDA, "moe_pack_mxfp4_scales", e);
}

int moe_quantize_fp8_block128(const float* w, int64_t batch, int32_t rows, int32_t K, uint8_t* q,
                              float* scales, void* stream) {
  if (!w || !q || !scales || batch < 1 || rows < 128 || K < 128 || rows % 128 || K % 128 || batch > 65535)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 16)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[3] = {w, q, scales};
  int dev = resolve_device(stream, ptrs, 3);
  if (dev < 0) return dev;
  DeviceGuard g(dev);
  return launch_quant_fp8(w, batch, rows, K, q, scales, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
