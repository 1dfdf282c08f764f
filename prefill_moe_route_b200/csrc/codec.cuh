// codec.cuh -- device helpers shared by the kernels: the specified routing
// sigmoid, power-of-two scale rules and the warp-level top-k routing of one
// token.
#pragma once
#include "internal.h"
#include "ptx.cuh"

namespace moe {

// Specified fp32 exponential: Cody & Waite (1980) reduction with a two-part
// ln 2, degree-7 Taylor polynomial in Horner form, scaling by 2^n through the
// exponent field.  Every operation is one round-to-nearest step (explicit
// _rn intrinsics, so nothing is contracted into an FMA).
__device__ __forceinline__ float exp_spec(float x) {
  const float LOG2E = 0x1.715476p+0f;
  const float C1 = 0x1.63p-1f;
  const float C2 = -0x1.bd0106p-13f;
  const float K2 = 0x1p-1f, K3 = 0x1.555556p-3f, K4 = 0x1.555556p-5f, K5 = 0x1.111112p-7f,
              K6 = 0x1.6c16c2p-10f, K7 = 0x1.a01a02p-13f;
  x = fminf(fmaxf(x, -87.0f), 88.0f);
  float n = rintf(__fmul_rn(x, LOG2E));
  float r = __fsub_rn(x, __fmul_rn(n, C1));
  r = __fsub_rn(r, __fmul_rn(n, C2));
  float p = K7;
  p = __fadd_rn(__fmul_rn(p, r), K6);
  p = __fadd_rn(__fmul_rn(p, r), K5);
  p = __fadd_rn(__fmul_rn(p, r), K4);
  p = __fadd_rn(__fmul_rn(p, r), K3);
  p = __fadd_rn(__fmul_rn(p, r), K2);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  float two_n = __int_as_float((static_cast<int>(n) + 127) << 23);
  return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float sigmoid_spec(float l) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_spec(-l)));
}

// 2^k as fp32 for k in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float exp2i(int k) {
  return k >= -126 ? __int_as_float((k + 127) << 23) : __int_as_float(0x00400000);
}

// floor(log2(a)) for finite a > 0, subnormals included.
__device__ __forceinline__ int floor_log2(float a) {
  uint32_t b = __float_as_uint(a);
  int ex = (b >> 23) & 0xFF;
  if (ex != 0) return ex - 127;
  uint32_t m = b & 0x7FFFFFu;
  return (31 - __clz(m)) - 149;
}

// Smallest k in [-126, 127] with amax <= 448 * 2^k (k = 0 for amax = 0).
__device__ __forceinline__ int pow2_e4m3_exp(float amax) {
  if (!(amax > 0.0f)) return 0;
  int E = floor_log2(amax);
  uint32_t b = __float_as_uint(amax);
  uint32_t mant;
  if (((b >> 23) & 0xFF) != 0) {
    mant = b & 0x7FFFFFu;
  } else {  // normalize the subnormal significand to 1.f form
    uint32_t m = b & 0x7FFFFFu;
    int sh = __clz(m) - 8;
    mant = (m << sh) & 0x7FFFFFu;
  }
  int k = (mant <= 0x600000u) ? E - 8 : E - 7;  // 448 = 1.75 * 2^8
  return max(-126, min(127, k));
}

// ---------------------------------------------------------------------------
// Warp-wide exclusive scan of one value per lane; returns the lane's prefix
// and sets *total.
__device__ __forceinline__ int warp_exclusive_scan(int v, int* total) {
  const int lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
    if (lane >= off) x += y;
  }
  *total = __shfl_sync(0xFFFFFFFFu, x, 31);
  return x - v;
}

// Orderable key of an fp32 value: a larger float gives a larger unsigned key
// (-0 is folded onto +0 first, so equal floats give equal keys).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  const uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Route one token with one warp: sigmoid of every logit, top-k of sigmoid +
// bias in k rounds (each the warp-wide maximum of the lanes' best candidates,
// a tie going to the lower expert ID), weights = selected sigmoids normalized
// to sum 1 (slot order) times the routed scale.  Lane j < k receives slot j's
// expert and weight.  ("glm53: FP8 mid hand-off", commit "per-row up/gate jobs
// at 4 rows": top-8 rounds; a tied round broken by expert ID.)
//
// Lane l holds experts l, l + 32, ... (KPER of them).  The sigmoids are
// computed in a rolled loop through `scratch` (2 * 32 * KPER words of shared
// memory owned by this warp), so the code stays short: a kernel runs it once,
// cold, and its instruction fetch is the larger cost.  A round is a warp
// max-reduction of the lanes' best keys and a min-reduction of the expert IDs
// among the lanes that hold that key.
template <int KPER>
__device__ __forceinline__ void route_token_warp_k(const float* logits_row, const float* bias, int E, int k,
                                                   float routed_scale, int* id_out, float* w_out,
                                                   uint32_t* scratch) {
  const int lane = threadIdx.x & 31;
  uint32_t* skey = scratch;                                   // [KPER][32] bias, then order keys
  float* ssig = reinterpret_cast<float*>(scratch + 32 * KPER);  // [KPER][32] logits, then sigmoids
  {  // every load in flight at once
    float lg[KPER], bs[KPER];
#pragma unroll
    for (int i = 0; i < KPER; ++i) {
      const int e = lane + 32 * i;
      lg[i] = e < E ? __ldg(logits_row + e) : 0.0f;
      bs[i] = (bias && e < E) ? __ldg(bias + e) : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < KPER; ++i) { ssig[i * 32 + lane] = lg[i]; skey[i * 32 + lane] = __float_as_uint(bs[i]); }
  }
#pragma unroll 1
  for (int i = 0; i < KPER; ++i) {
    const int e = lane + 32 * i;
    uint32_t key = 0u;   // below every finite key: never selected while k <= E
    float sg = 0.0f;
    if (e < E) {
      sg = sigmoid_spec(ssig[i * 32 + lane]);
      key = float_order_key(bias ? __fadd_rn(sg, __uint_as_float(skey[i * 32 + lane])) : sg);
    }
    skey[i * 32 + lane] = key;
    ssig[i * 32 + lane] = sg;
  }
  __syncwarp();
  uint32_t key[KPER];
#pragma unroll
  for (int i = 0; i < KPER; ++i) key[i] = skey[i * 32 + lane];
  float denom = 0.0f;
  int my_id = -1;
  float my_s = 0.0f;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < KPER; ++i)
      if (key[i] > best) { best = key[i]; bi = i; }   // strict: the lower expert of a tie stays
    const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, best);
    const uint32_t emin = __reduce_min_sync(0xFFFFFFFFu, best == kmax ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu);
    if ((int)(emin & 31u) == lane) {
#pragma unroll
      for (int i = 0; i < KPER; ++i)
        if (i == (int)(emin >> 5)) key[i] = 0u;   // taken
    }
    const float sv = ssig[emin];                  // (emin >> 5) * 32 + (emin & 31)
    denom = __fadd_rn(denom, sv);  // slot order
    if (lane == j) { my_id = (int)emin; my_s = sv; }
  }
  if (lane < k) {
    *id_out = my_id;
    *w_out = __fmul_rn(__fdiv_rn(my_s, denom), routed_scale);
  }
  __syncwarp();   // scratch reads done before the warp reuses it
}

// A token routed by the caller: lane j < k takes slot j.  An expert ID
// outside [0, E) is recorded in the status word (ST_BAD_INPUT) and replaced
// by expert 0 with weight 0, the same way on every CTA, so the call still
// runs to its end with in-range indices.
__device__ __forceinline__ void take_routed_token(const int32_t* ids_row, const float* w_row, int E, int k,
                                                  int* id_out, float* w_out, int32_t* status) {
  const int lane = threadIdx.x & 31;
  if (lane < k) {
    int id = __ldg(ids_row + lane);
    float w = __ldg(w_row + lane);
    if (id < 0 || id >= E) {
      atomicOr(status, ST_BAD_INPUT);
      id = 0;
      w = 0.0f;
    }
    *id_out = id;
    *w_out = w;
  }
}

// scratch: 2 * kMaxE words of shared memory owned by the calling warp.
__device__ __forceinline__ void route_token_warp(const float* logits_row, const float* bias, int E, int k,
                                                 float routed_scale, int* id_out, float* w_out, uint32_t* scratch) {
  if (E <= 256) route_token_warp_k<8>(logits_row, bias, E, k, routed_scale, id_out, w_out, scratch);
  else route_token_warp_k<kMaxE / 32>(logits_row, bias, E, k, routed_scale, id_out, w_out, scratch);
}

}  // namespace moe
