// route.cu -- step 1 of the MoE call: sigmoid+bias top-k routing (a warp per
// token), quantization of the token's activation row, and -- in the CTA that
// finishes last -- the stable expert-major sort of the (token, slot) pairs.
//
// Routing follows "glm53: FP8 mid hand-off" (commit "per-row up/gate jobs at
// 4 rows"): top-k rounds, each taking the warp-wide maximum of the lanes'
// best candidates; a tie is broken by the lower expert ID.  The weights are
// the selected sigmoids normalized to sum 1, times the routed scale.
// Activation quantization: MXFP4 (OCP MX v1.0: E8M0 scale
// 2^(floor(log2 amax) - 2) per 32, E2M1 RNE saturating) for MXFP4 weights --
// the "A4W4" arm of "IQ2R: load GLM-5.3 packed MoE checkpoints"; E4M3 with a
// power-of-two scale per 128 for block-FP8 weights.
// The sort is the expert-major grouping of "glm53_flash: score a verify
// request's index tiles once": pairs grouped by expert, ascending pair id
// inside an expert.
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
constexpr int kRouteWarps = 8;

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

constexpr int kBatch = 8;  // 32-pair steps whose ids are loaded together

// Stable counting sort of the pairs by expert plus the per-expert tile
// prefixes the grouped GEMMs schedule from.  Runs in one CTA: each warp owns a
// contiguous range of pairs; ranks inside a 32-pair step come from the match
// mask, so the order inside an expert is ascending pair id.
__device__ void align_pairs(const RouteParams& p) {
  __shared__ int wcnt[kRouteWarps][kMaxE];
  const int E = p.E, P = p.M * p.topk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = ((P + kRouteWarps - 1) / kRouteWarps + 31) & ~31;
  const int beg = warp * chunk, end = min(P, beg + chunk);

  for (int i = threadIdx.x; i < kRouteWarps * kMaxE; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  // phase 1: per-warp expert counts over the warp's pair range
  for (int base = beg; base < end; base += 32 * kBatch) {
    int ids[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int pi = base + 32 * b + lane;
      ids[b] = pi < end ? __ldcg(p.topk_ids + pi) : -1;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, ids[b]);
      if (ids[b] >= 0 && lane == __ffs(peers) - 1) wcnt[warp][ids[b]] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  // phase 2 (warp 0): totals, exclusive prefixes, tile counts, per-warp starts
  if (warp == 0) {
    constexpr int kPer = kMaxE / 32;
    const int per = (E + 31) / 32;
    int c[kPer], t1[kPer], t2[kPer];
    int s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane * per + i;
      int cnt = 0;
      if (i < per && e < E)
        for (int w = 0; w < kRouteWarps; ++w) cnt += wcnt[w][e];
      c[i] = cnt;
      t1[i] = (cnt + p.nt1 - 1) / p.nt1;
      t2[i] = (cnt + p.nt2 - 1) / p.nt2;
      s0 += c[i]; s1 += t1[i]; s2 += t2[i];
    }
    int tot0, tot1, tot2;
    int o0 = warp_exclusive_scan(s0, &tot0);
    int o1 = warp_exclusive_scan(s1, &tot1);
    int o2 = warp_exclusive_scan(s2, &tot2);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane * per + i;
      if (i < per && e < E) {
        p.counts[e] = c[i];
        p.offsets[e] = o0;
        p.tiles1[e] = o1;
        p.tiles2[e] = o2;
        int run = o0;
        for (int w = 0; w < kRouteWarps; ++w) {
          const int cw = wcnt[w][e];
          wcnt[w][e] = run;
          run += cw;
        }
      }
      o0 += c[i]; o1 += t1[i]; o2 += t2[i];
    }
    if (lane == 0) {
      p.offsets[E] = tot0;
      p.tiles1[E] = tot1;
      p.tiles2[E] = tot2;
    }
  }
  __syncthreads();
  // phase 3: scatter
  const unsigned lt = (1u << lane) - 1u;
  for (int base = beg; base < end; base += 32 * kBatch) {
    int ids[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int pi = base + 32 * b + lane;
      ids[b] = pi < end ? __ldcg(p.topk_ids + pi) : -1;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int pi = base + 32 * b + lane;
      const int e = ids[b];
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      if (e >= 0) {
        const int pos = wcnt[warp][e] + __popc(peers & lt);
        p.sorted_pairs[pos] = pi;
        p.inv[pi] = pos;
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) wcnt[warp][e] += __popc(peers);
      __syncwarp();
    }
  }
}

// One CTA per token: warp 0 routes the token, all warps quantize its row.
__global__ void __launch_bounds__(kRouteWarps * 32)
k_route_quant_align(const RouteParams p) {
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int E = p.E, k = p.topk;

  if (warp == 0) {
    // ---- routing: lane owns experts lane, lane+32, ...
    constexpr int kPer = kMaxE / 32;
    float s_loc[kPer], sel_loc[kPer];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      s_loc[i] = 0.0f;
      sel_loc[i] = -INFINITY;
      if (e < E) {
        const float s = sigmoid_spec(__ldg(p.logits + (size_t)t * E + e));
        s_loc[i] = s;
        sel_loc[i] = p.bias ? __fadd_rn(s, __ldg(p.bias + e)) : s;
      }
    }
    float denom = 0.0f;
    int my_id = -1;
    float my_s = 0.0f;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int be = 0x7FFFFFFF;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && sel_loc[i] > bv) { bv = sel_loc[i]; be = e; }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
        const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
        if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
      }
      // the owner lane marks the pick and broadcasts its sigmoid
      float sv = 0.0f;
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (lane + 32 * i == be) { taken |= 1u << i; sv = s_loc[i]; }
      sv = __shfl_sync(0xFFFFFFFFu, sv, be & 31);
      denom = __fadd_rn(denom, sv);  // slot order
      if (lane == j) { my_id = be; my_s = sv; }
    }
    if (lane < k) {
      p.topk_ids[(size_t)t * k + lane] = my_id;
      p.topk_w[(size_t)t * k + lane] = __fmul_rn(__fdiv_rn(my_s, denom), p.routed_scale);
    }
  }

  // ---- activation quantization of row t (all warps; loads first)
  if (p.x) {
    const uint16_t* xr = p.x + (size_t)t * p.H;
    if (p.wfmt == MOE_W_MXFP4) {
      uint8_t* xs = static_cast<uint8_t*>(p.xs) + (size_t)t * (p.H / 32);
      uint8_t* xq = p.xq + (size_t)t * (p.H / 2);
      for (int b = threadIdx.x; b < p.H / 32; b += blockDim.x) {  // one 32-element block per thread
        const uint4* src = reinterpret_cast<const uint4*>(xr + b * 32);
        uint4 u[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) u[c] = __ldg(src + c);
        float v[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[c * 8 + 2 * i] = __uint_as_float(w[i] << 16);
            v[c * 8 + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
          }
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
        int code = 0;
        if (amax > 0.0f) code = max(0, min(254, floor_log2(amax) - 2 + 127));
        const float inv = exp2i(127 - code);
        uint32_t out[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(v[c * 8 + i], inv);
          out[c] = cvt_e2m1x8(f);
        }
        reinterpret_cast<uint4*>(xq + b * 16)[0] = make_uint4(out[0], out[1], out[2], out[3]);
        xs[b] = static_cast<uint8_t>(code);
      }
    } else {
      float* xs = static_cast<float*>(p.xs) + (size_t)t * (p.H / 128);
      uint8_t* xq = p.xq + (size_t)t * p.H;
      const int nb = p.H / 128;
      for (int b0 = warp; b0 < nb; b0 += 4 * kRouteWarps) {  // a warp per 128-element block
        uint2 u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int b = b0 + i * kRouteWarps;
          if (b < nb) u[i] = __ldg(reinterpret_cast<const uint2*>(xr + b * 128) + lane);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int b = b0 + i * kRouteWarps;
          if (b >= nb) break;
          const float v[4] = {__uint_as_float(u[i].x << 16), __uint_as_float(u[i].x & 0xFFFF0000u),
                              __uint_as_float(u[i].y << 16), __uint_as_float(u[i].y & 0xFFFF0000u)};
          float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
          const int ke = pow2_e4m3_exp(amax);
          const float inv = exp2i(-ke);
          const uint32_t q = cvt_e4m3x4(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv), __fmul_rn(v[2], inv),
                                        __fmul_rn(v[3], inv));
          reinterpret_cast<uint32_t*>(xq + b * 128)[lane] = q;
          if (lane == 0) xs[b] = exp2i(ke);
        }
      }
    }
  }

  if (!p.do_align) return;
  // ---- the last CTA to finish sorts the pairs
  __shared__ int is_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    int old = atomicAdd(p.status + 1, 1);
    is_last = (old == (int)gridDim.x - 1);
    if (is_last) p.status[1] = 0;  // leave the counter at zero for the next call
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  align_pairs(p);
}

}  // namespace moe
