// route.cu -- step 1 of the MoE call: sigmoid+bias top-k routing (a warp per
// token), quantization of the token's activation row, and the stable
// expert-major sort of the (token, slot) pairs: counts per (chunk of tokens,
// expert) during routing, their prefixes in the route CTA that finishes last,
// and a scatter kernel with one CTA per chunk.
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

// Block-wide exclusive scan of one value per thread (blockDim.x = 256);
// returns the thread's prefix and sets *total (all threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* total) {
  __shared__ int wsum[kRouteWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int wt;
  const int x = warp_exclusive_scan(v, &wt);
  if (lane == 0) wsum[warp] = wt;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kRouteWarps; ++w) {
    if (w < warp) base += wsum[w];
    tot += wsum[w];
  }
  __syncthreads();   // wsum may be reused by the next scan
  *total = tot;
  return base + x;
}

// Totals of the sort, run by the route CTA that finishes last.  The route
// CTAs counted their pairs per (chunk of tokens, expert) with atomics; here
// each expert's chunk counts become exclusive prefixes over the chunks (the
// scatter kernel adds the expert's offset), and the per-expert totals become
// counts, offsets and the token-tile prefixes the grouped GEMMs schedule from.
__device__ void align_totals(const RouteParams& p) {
  const int E = p.E, nch = p.nchunks;
  // thread i owns experts 2i and 2i + 1 (E <= 512); the chunk counts of both
  // are loaded 16 chunks at a time so their latencies overlap
  int c[2] = {0, 0};
  const int e0 = 2 * threadIdx.x;
  for (int ch0 = 0; ch0 < nch; ch0 += 16) {
    int v[2][16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u)
        v[u][i] = (ch0 + i < nch && e0 + u < E) ? __ldcg(p.chunk_cnt + (size_t)(ch0 + i) * E + e0 + u) : 0;
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (ch0 + i < nch && e0 + u < E) p.chunk_cnt[(size_t)(ch0 + i) * E + e0 + u] = c[u];
        c[u] += v[u][i];
      }
  }
  const int t1a = (c[0] + p.nt1 - 1) / p.nt1, t1b = (c[1] + p.nt1 - 1) / p.nt1;
  const int t2a = (c[0] + p.nt2 - 1) / p.nt2, t2b = (c[1] + p.nt2 - 1) / p.nt2;
  int tot0, tot1, tot2;
  const int o0 = block_exclusive_scan(c[0] + c[1], &tot0);
  const int o1 = block_exclusive_scan(t1a + t1b, &tot1);
  const int o2 = block_exclusive_scan(t2a + t2b, &tot2);
  if (e0 < E) {
    p.counts[e0] = c[0]; p.offsets[e0] = o0; p.tiles1[e0] = o1; p.tiles2[e0] = o2;
  }
  if (e0 + 1 < E) {
    p.counts[e0 + 1] = c[1]; p.offsets[e0 + 1] = o0 + c[0]; p.tiles1[e0 + 1] = o1 + t1a; p.tiles2[e0 + 1] = o2 + t2a;
  }
  if (threadIdx.x == 0) {
    p.offsets[E] = tot0;
    p.tiles1[E] = tot1;
    p.tiles2[E] = tot2;
  }
}

// Stable scatter of one chunk of pairs (grid: one CTA per chunk).  The chunk's
// pairs land at offsets[e] + (pairs of expert e in earlier chunks) + (earlier
// pairs of expert e in this chunk): grouped by expert, ascending pair id
// inside an expert ("glm53_flash: score a verify request's index tiles once",
// expert-major order).  Each warp owns a contiguous range of the chunk; ranks
// inside a 32-pair step come from the match mask.  The CTA leaves its row of
// chunk prefixes at zero for the next call's counting.
__global__ void __launch_bounds__(kRouteWarps * 32) k_align_scatter(const RouteParams p) {
  __shared__ int wcnt[kRouteWarps][kMaxE];
  pdl_wait();                 // routing, counts and prefixes of this call are complete
  pdl_launch_dependents();
  const int E = p.E, P = p.M * p.topk;
  const int ch = blockIdx.x;
  const int cbeg = ch * p.chunk_pairs, cend = min(P, cbeg + p.chunk_pairs);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int span = cend - cbeg;
  const int chunk = ((span + kRouteWarps - 1) / kRouteWarps + 31) & ~31;
  const int beg = cbeg + warp * chunk, end = min(cend, beg + chunk);

  for (int i = threadIdx.x; i < kRouteWarps * kMaxE; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  // per-warp expert counts over the warp's range
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
  // per-warp starting positions of each expert
  int32_t* rel = p.chunk_cnt + (size_t)ch * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = __ldcg(p.offsets + e) + __ldcg(rel + e);
    rel[e] = 0;
#pragma unroll
    for (int w = 0; w < kRouteWarps; ++w) {
      const int cw = wcnt[w][e];
      wcnt[w][e] = run;
      run += cw;
    }
  }
  __syncthreads();
  // scatter
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
        p.sorted_w[pos] = __ldcg(p.topk_w + pi);
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) wcnt[warp][e] += __popc(peers);
      __syncwarp();
    }
  }
}

// GEMM1's operand in sorted-pair order, so that a token tile is one 2-D
// tile copy per pipeline stage: the quantized row of each pair's token, and
// its scales packed per (token tile, 128-column chunk of H) in the order the
// tensor cores' scale-factor copy reads them (512-byte blocks, the tile's row
// m (0..nt-1) at byte 16 * (m % 32) + 4 * (m / 32), its four per-32 scales in
// column order).  MXFP4 tokens: the four E8M0 codes of the chunk; E4M3 tokens:
// the power-of-two scale of the chunk as an E8M0 code, repeated for the four
// sub-blocks.
__global__ void __launch_bounds__(256) k_pack_operand(const RouteParams p) {
  pdl_wait();                 // the sort of this call is complete
  pdl_launch_dependents();
  const int P = p.M * p.topk, nch = p.H / 128;
  const bool mx = p.wfmt == MOE_W_MXFP4;
  const int rowv = nch * (mx ? 4 : 8);   // 16-byte words of a quantized row
  const int lane = threadIdx.x & 31;
  // one warp per sorted pair: its token's quantized row, 16 bytes per lane per step
  for (int pos = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; pos < P; pos += (gridDim.x * blockDim.x) >> 5) {
    const int pair = __ldcg(p.sorted_pairs + pos);
    const int t = pair / p.topk, e = __ldcg(p.topk_ids + pair);
    const int rel = pos - __ldcg(p.offsets + e);
    const int tile = __ldcg(p.tiles1 + e) + rel / p.nt1, m = rel % p.nt1;
    const uint4* src = reinterpret_cast<const uint4*>(p.xq) + (size_t)t * rowv;
    uint4* dst = reinterpret_cast<uint4*>(p.xg) + (size_t)pos * rowv;
    for (int i = lane; i < rowv; i += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i + 32 * u < rowv) v[u] = __ldcg(src + i + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i + 32 * u < rowv) dst[i + 32 * u] = v[u];
    }
    for (int ch = lane; ch < nch; ch += 32) {
      uint32_t sc;
      if (mx)
        sc = __ldcg(reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(p.xs) + (size_t)t * (p.H / 32)) + ch);
      else
        sc = rep4((__float_as_uint(__ldcg(static_cast<const float*>(p.xs) + (size_t)t * nch + ch)) >> 23) & 0xFFu);
      p.bsf[((size_t)tile * nch + ch) * 128 + 4 * (m % 32) + m / 32] = sc;
    }
  }
}

// Up to kRouteWarps tokens per CTA (the launch picks the grid; the CTA's
// share is ceil(M / grid)): warp w routes the CTA's token w, then all warps
// quantize the CTA's rows (loads first).
__global__ void __launch_bounds__(kRouteWarps * 32)
k_route_quant_align(const RouteParams p) {
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tpc = (p.M + (int)gridDim.x - 1) / (int)gridDim.x;   // <= kRouteWarps by the launch
  const int t0 = blockIdx.x * tpc;
  const int rows = min(tpc, p.M - t0);   // <= 0 only for a CTA past the last token: it still counts in
  const int E = p.E, k = p.topk;

  __shared__ uint32_t rscratch[kRouteWarps][2 * kMaxE];
  if (warp < rows) {
    const int t = t0 + warp;
    if (p.ids_in)
      take_routed_token(p.ids_in + (size_t)t * k, p.w_in + (size_t)t * k, E, k, p.topk_ids + (size_t)t * k + lane,
                        p.topk_w + (size_t)t * k + lane, p.status);
    else
      route_token_warp(p.logits + (size_t)t * E, p.bias, E, k, p.routed_scale,
                       p.topk_ids + (size_t)t * k + lane, p.topk_w + (size_t)t * k + lane, rscratch[warp]);
    // count the token's pairs for its chunk (the ids were written by this lane)
    if (p.do_align && lane < k) atomicAdd(p.chunk_cnt + (size_t)(t / p.chunk_tokens) * E + p.topk_ids[(size_t)t * k + lane], 1);
  }

  // ---- activation quantization of the CTA's rows
  if (p.x) {
    if (p.wfmt == MOE_W_MXFP4) {
      const int nb = p.H / 32;
      for (int idx = threadIdx.x; idx < rows * nb; idx += blockDim.x) {  // one 32-element block per thread
        const int t = t0 + idx / nb, b = idx % nb;
        const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H + b * 32);
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
        reinterpret_cast<uint4*>(p.xq + (size_t)t * (p.H / 2) + b * 16)[0] = make_uint4(out[0], out[1], out[2], out[3]);
        static_cast<uint8_t*>(p.xs)[(size_t)t * nb + b] = static_cast<uint8_t>(code);
      }
    } else {
      // a half-warp per 128-element block (16 bytes per lane), four blocks per
      // half-warp in flight.  The loop runs on the warp's first block so that
      // both halves make the same trips (the shuffles take the whole warp).
      const int nb = p.H / 128, hw = lane >> 4, hl = lane & 15;
      const int nblk = rows * nb;
      for (int w0 = 2 * warp; w0 < nblk; w0 += 8 * kRouteWarps) {
        const int b0 = w0 + hw;
        uint4 u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int bb = b0 + i * 2 * kRouteWarps;
          if (bb < nblk)
            u[i] = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)(t0 + bb / nb) * p.H + (bb % nb) * 128) + hl);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          // every lane takes part in the shuffles; lanes past the last block drop their result
          const int bb = b0 + i * 2 * kRouteWarps;
          const bool live = bb < nblk;
          const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
          float v[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
          }
          float amax = 0.0f;
          if (live) {
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
          }
#pragma unroll
          for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
          if (!live) continue;
          const int t = t0 + bb / nb, b = bb % nb;
          const int ke = pow2_e4m3_exp(amax);
          const float inv = exp2i(-ke);
          const uint2 q = make_uint2(
              cvt_e4m3x4(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv), __fmul_rn(v[2], inv), __fmul_rn(v[3], inv)),
              cvt_e4m3x4(__fmul_rn(v[4], inv), __fmul_rn(v[5], inv), __fmul_rn(v[6], inv), __fmul_rn(v[7], inv)));
          reinterpret_cast<uint2*>(p.xq + (size_t)t * p.H + b * 128)[hl] = q;
          if (hl == 0) static_cast<float*>(p.xs)[(size_t)t * nb + b] = exp2i(ke);
        }
      }
    }
  }

  if (!p.do_align) return;
  // ---- the last CTA to finish turns the chunk counts into the sort's totals
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
  align_totals(p);
}

}  // namespace moe
