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
#include "codec.cuh"

namespace moe {

constexpr int kRouteWarps = 8;

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

  __shared__ uint32_t rscratch[2 * kMaxE];
  if (warp == 0) {
    if (p.ids_in)
      take_routed_token(p.ids_in + (size_t)t * k, p.w_in + (size_t)t * k, E, k, p.topk_ids + (size_t)t * k + lane,
                        p.topk_w + (size_t)t * k + lane, p.status);
    else
      route_token_warp(p.logits + (size_t)t * E, p.bias, E, k, p.routed_scale,
                       p.topk_ids + (size_t)t * k + lane, p.topk_w + (size_t)t * k + lane, rscratch);
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
