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
// Lane l holds experts l, l + 32, ...  It sorts them once (a bitonic network in
// registers) by (key descending, expert ascending), so its best remaining
// candidate is always its head; a round is then a warp max-reduction of the
// heads' keys and a min-reduction of the expert IDs among the lanes that hold
// that key, and the winning lane shifts its list by one.
template <int KPER>
__device__ __forceinline__ void route_token_warp_k(const float* logits_row, const float* bias, int E, int k,
                                                   float routed_scale, int* id_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  uint32_t key[KPER];
  int ex[KPER];
  float sv[KPER];
#pragma unroll
  for (int i = 0; i < KPER; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0u;                       // below every finite key: never selected while k <= E
    ex[i] = 0x7FFFFFFF;
    sv[i] = 0.0f;
    if (e < E) {
      const float s = sigmoid_spec(__ldg(logits_row + e));
      sv[i] = s;
      ex[i] = e;
      key[i] = float_order_key(bias ? __fadd_rn(s, __ldg(bias + e)) : s);
    }
  }
  // bitonic sort, descending by key, ascending by expert on equal keys
#pragma unroll
  for (int k2 = 2; k2 <= KPER; k2 <<= 1)
#pragma unroll
    for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1)
#pragma unroll
      for (int i = 0; i < KPER; ++i) {
        const int l = i ^ j2;
        if (l > i) {
          const bool l_first = key[l] > key[i] || (key[l] == key[i] && ex[l] < ex[i]);
          const bool swap = ((i & k2) == 0) ? l_first : !l_first;
          if (swap) {
            const uint32_t tk = key[i]; key[i] = key[l]; key[l] = tk;
            const int te = ex[i]; ex[i] = ex[l]; ex[l] = te;
            const float ts = sv[i]; sv[i] = sv[l]; sv[l] = ts;
          }
        }
      }
  float denom = 0.0f;
  int my_id = -1;
  float my_s = 0.0f;
  for (int j = 0; j < k; ++j) {
    const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, key[0]);
    const uint32_t emin = __reduce_min_sync(0xFFFFFFFFu, key[0] == kmax ? (uint32_t)ex[0] : 0xFFFFFFFFu);
    const float s = __shfl_sync(0xFFFFFFFFu, sv[0], (int)(emin & 31u));
    denom = __fadd_rn(denom, s);  // slot order
    if (lane == j) { my_id = (int)emin; my_s = s; }
    if ((uint32_t)ex[0] == emin) {  // the winner advances to its next candidate
#pragma unroll
      for (int i = 0; i + 1 < KPER; ++i) { key[i] = key[i + 1]; ex[i] = ex[i + 1]; sv[i] = sv[i + 1]; }
      key[KPER - 1] = 0u;
      ex[KPER - 1] = 0x7FFFFFFF;
    }
  }
  if (lane < k) {
    *id_out = my_id;
    *w_out = __fmul_rn(__fdiv_rn(my_s, denom), routed_scale);
  }
}

__device__ __forceinline__ void route_token_warp(const float* logits_row, const float* bias, int E, int k,
                                                 float routed_scale, int* id_out, float* w_out) {
  if (E <= 256) route_token_warp_k<8>(logits_row, bias, E, k, routed_scale, id_out, w_out);
  else route_token_warp_k<kMaxE / 32>(logits_row, bias, E, k, routed_scale, id_out, w_out);
}

}  // namespace moe
