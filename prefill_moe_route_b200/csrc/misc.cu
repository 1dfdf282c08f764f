// misc.cu -- the deterministic routing-weighted combine, the offline weight
// quantizers, and host launch helpers for the route and combine kernels.
#include "internal.h"
#include "ptx.cuh"

namespace moe {

__global__ void k_route_quant_align(const RouteParams p);  // route.cu
__global__ void k_align_scatter(const RouteParams p);      // route.cu
__global__ void k_pack_operand(const RouteParams p);       // route.cu

// out[t, h] = bf16( sum_j yw[slot(t, j), h] ), j ascending, fp32, where yw is
// GEMM2's output already weighted (bf16(w_j * y)).  One thread owns 16
// consecutive h of one token (two 16-byte loads per slot, all slots' loads in
// flight before the sum): no atomics, run-to-run identical ("IQ2R: load
// GLM-5.3 packed MoE checkpoints", benchmark notes: interleaved down /
// reduction; batched reduction).
__global__ void __launch_bounds__(256) k_combine(const CombineParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.y;
  const int h0 = (blockIdx.x * blockDim.x + threadIdx.x) * 16;
  if (h0 >= p.H) return;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
  for (int j0 = 0; j0 < p.topk; j0 += 8) {
    int r[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j0 + j < p.topk) r[j] = __ldcg(p.inv + (size_t)t * p.topk + j0 + j);
    uint4 v[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j0 + j < p.topk) {
        const uint4* src = reinterpret_cast<const uint4*>(p.yw + (size_t)r[j] * p.H + h0);
        v[j][0] = __ldcs(src);
        v[j][1] = __ldcs(src + 1);
      }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j0 + j < p.topk) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t w4[4] = {v[j][hh].x, v[j][hh].y, v[j][hh].z, v[j][hh].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[8 * hh + 2 * i] += __uint_as_float(w4[i] << 16);
            acc[8 * hh + 2 * i + 1] += __uint_as_float(w4[i] & 0xFFFF0000u);
          }
        }
      }
    }
  }
  if (p.out_f32) {   // a tensor-parallel rank's partial: the ranks' sums meet in an all-reduce
    float4* dst = reinterpret_cast<float4*>(p.out_f32 + (size_t)t * p.H + h0);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    return;
  }
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
  uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)t * p.H + h0);
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// bf16 (round to nearest even) of n floats, 8 per thread (n % 8 == 0).
__global__ void __launch_bounds__(256) k_round_bf16(const float* __restrict__ in, uint16_t* __restrict__ out,
                                                    int64_t n8) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = __ldcs(reinterpret_cast<const float4*>(in) + 2 * i);
  const float4 b = __ldcs(reinterpret_cast<const float4*>(in) + 2 * i + 1);
  reinterpret_cast<uint4*>(out)[i] =
      make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

__device__ __forceinline__ float pow2_of(int k) {
  return k >= -126 ? __int_as_float((k + 127) << 23) : __int_as_float(0x00400000);
}

// OCP MX v1.0 conversion of one 32-element block per thread: shared scale
// 2^(floor(log2 amax) - 2) stored as E8M0, elements E2M1 RNE saturating.
__global__ void __launch_bounds__(256) k_quant_mxfp4(const float* __restrict__ w, int64_t nblocks,
                                                     uint8_t* __restrict__ q, uint8_t* __restrict__ s) {
  const int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const float4* src = reinterpret_cast<const float4*>(w + b * 32);
  float v[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 f = __ldg(src + i);
    v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  int code = 0;
  if (amax > 0.0f) {
    const uint32_t bits = __float_as_uint(amax);
    const int ex = (bits >> 23) & 0xFF;
    const int fl = ex ? ex - 127 : (31 - __clz(bits & 0x7FFFFFu)) - 149;
    code = max(0, min(254, fl - 2 + 127));
  }
  const float inv = pow2_of(127 - code);
  uint32_t out[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float f[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(v[c * 8 + i], inv);
    out[c] = cvt_e2m1x8(f);
  }
  reinterpret_cast<uint4*>(q + b * 16)[0] = make_uint4(out[0], out[1], out[2], out[3]);
  s[b] = static_cast<uint8_t>(code);
}

// Row-major E8M0 scales -> tensor-core scale-factor blocks, one 4-scale word
// per thread: word (b, r, g) of [batch][rows][K/128] goes to block
// (b, r / 128, g), byte 16 * (r % 32) + 4 * ((r % 128) / 32).
__global__ void __launch_bounds__(256) k_pack_mx_scales(const uint32_t* __restrict__ s, int64_t nwords, int rows,
                                                        int g_per_row, uint32_t* __restrict__ out) {
  const int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (w >= nwords) return;
  const int g = (int)(w % g_per_row);
  const int64_t br = w / g_per_row;            // b * rows + r
  const int r = (int)(br % rows);
  const int64_t b = br / rows;
  const int64_t blk = (b * (rows / 128) + r / 128) * g_per_row + g;
  out[blk * 128 + 4 * (r % 32) + (r % 128) / 32] = __ldg(s + w);
}

// 128x128 block FP8: one CTA per block; scale = amax / 448 (fp32), 1 for an
// all-zero block; q = E4M3(w / scale) RNE saturating.
__global__ void __launch_bounds__(256) k_quant_fp8_block128(const float* __restrict__ w, int rows, int K,
                                                            uint8_t* __restrict__ q, float* __restrict__ s) {
  __shared__ float red[8];
  const int bk = blockIdx.x, br = blockIdx.y, bb = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t base = ((size_t)bb * rows + (size_t)br * 128) * K + (size_t)bk * 128;
  float4 v[16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = warp + 8 * i;
    v[i] = __ldg(reinterpret_cast<const float4*>(w + base + (size_t)r * K) + lane);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = warp + 8 * i;
    const uint32_t qv = cvt_e4m3x4(__fdiv_rn(v[i].x, sc), __fdiv_rn(v[i].y, sc), __fdiv_rn(v[i].z, sc),
                                   __fdiv_rn(v[i].w, sc));
    reinterpret_cast<uint32_t*>(q + base + (size_t)r * K)[lane] = qv;
  }
  if (threadIdx.x == 0) s[((size_t)bb * (rows / 128) + br) * (K / 128) + bk] = sc;
}

// ---------------------------------------------------------------------------
static cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

cudaError_t launch_route(const RouteParams& p, cudaStream_t st) {
  // tokens per CTA: one while M <= 128 (M = 16: 19.8 against 23.4 us for the
  // route, sort and packing launches), eight above (M = 1024: 32.7 us with
  // eight, 39.5 with four)
  const int tpc = p.M <= 128 ? 1 : 8;
  k_route_quant_align<<<(p.M + tpc - 1) / tpc, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_align(const RouteParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nchunks);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_align_scatter, p);
}

cudaError_t launch_pack_bsf(const RouteParams& p, int num_sms, cudaStream_t st) {
  const int64_t warps = (int64_t)p.M * p.topk;          // one warp per sorted pair
  const int64_t want = (warps + 7) / 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(want < 16 * num_sms ? want : 16 * num_sms));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_pack_operand, p);
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.H / 16 + 255) / 256, p.M);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_combine, p);
}

cudaError_t launch_round_bf16(const float* in, uint16_t* out, int64_t n, cudaStream_t st) {
  const int64_t n8 = n / 8;
  k_round_bf16<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(in, out, n8);
  return cudaGetLastError();
}

cudaError_t launch_quant_mxfp4(const float* w, int64_t nblocks, uint8_t* q, uint8_t* s, cudaStream_t st) {
  const int64_t grid = (nblocks + 255) / 256;
  k_quant_mxfp4<<<(unsigned)grid, 256, 0, st>>>(w, nblocks, q, s);
  return cudaGetLastError();
}

cudaError_t launch_pack_mx_scales(const uint8_t* s, int64_t batch, int rows, int K, uint8_t* out,
                                  cudaStream_t st) {
  const int64_t nwords = batch * rows * (int64_t)(K / 128);
  k_pack_mx_scales<<<(unsigned)((nwords + 255) / 256), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(s), nwords,
                                                                     rows, K / 128, reinterpret_cast<uint32_t*>(out));
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const float* w, int64_t batch, int rows, int K, uint8_t* q, float* s,
                             cudaStream_t st) {
  k_quant_fp8_block128<<<dim3(K / 128, rows / 128, (unsigned)batch), 256, 0, st>>>(w, rows, K, q, s);
  return cudaGetLastError();
}

}  // namespace moe
