// probe.cu -- the tensor cores' measured throughput for the MMA kinds the
// GEMMs issue, the denominator of the call's tensor fraction.
//
// One CTA per SM (its shared memory keeps a second one out); one thread issues
// `iters` blocks of four M = 128, N = 128 MMAs of one kind back to back into
// one TMEM accumulator, on K-major 128-byte-swizzled operands that stay in
// shared memory (every value 1.0, every block scale 2^0), and times them with
// %globaltimer and the SM clock up to the completion of the last one.  Nothing
// else runs in the kernel, so the figure is the pipe's issue-limited peak for
// that kind on this part and clock.  The pages check their counters against a
// workload whose answer is known ("IQ2R: load GLM-5.3 packed MoE checkpoints
// with TP slicing", the single-GPU MoE result sections); this is the same idea
// for the tensor side.
#include "codec.cuh"

namespace moe {

constexpr int kProbeMaxCtas = 1024;
__device__ unsigned long long g_probe[kProbeMaxCtas][2];   // per CTA: ns, SM cycles (0: the wait ran out)

constexpr int kProbeA = 128 * 128, kProbeB = 128 * 128;
constexpr int kProbeSmem = 120 * 1024;   // more than half of an SM's shared memory: one CTA per SM

// MACs of one instruction: K = 32 (8-bit), 64 (4-bit), 16 (bf16) per 128-byte row
__host__ __device__ constexpr double probe_macs_per_mma(int kind) {
  return 128.0 * 128.0 * (kind == MOE_PROBE_FP8 ? 32 : kind == MOE_PROBE_FP4 ? 64 : 16);
}

template <int KIND>
__global__ void __launch_bounds__(128, 1) k_tensor_probe(int iters, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sfa = smem + kProbeA + kProbeB;   // FP4: two 512-byte scale blocks per operand
  uint8_t* sfb = sfa + 1024;
  uint64_t* done = reinterpret_cast<uint64_t*>(sfb + 1024);
  uint32_t* holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  const int warp = threadIdx.x >> 5;
  // 1.0 as E4M3 (0x38), as two E2M1 codes (0x22), as bf16 (0x3F80)
  const uint32_t one = KIND == MOE_PROBE_FP8 ? 0x38383838u : KIND == MOE_PROBE_FP4 ? 0x22222222u : 0x3F803F80u;
  for (int i = threadIdx.x; i < (kProbeA + kProbeB) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(smem)[i] = one;
  for (int i = threadIdx.x; i < 2048 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sfa)[i] = 0x7F7F7F7Fu;
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (warp == 1) { tmem_alloc(holder, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;   // accumulator in columns 0..127, FP4 scales from column 128

  if (threadIdx.x == 0) {
    constexpr uint32_t IDESC = KIND == MOE_PROBE_FP8 ? idesc_f8f6f4(FMT8_E4M3, FMT8_E4M3, 128, 128)
                             : KIND == MOE_PROBE_FP4 ? idesc_block_scaled(FMT4_E2M1, FMT4_E2M1, 128)
                                                     : idesc_bf16(128);
    const uint32_t a_base = smem_u32(smem), b_base = a_base + kProbeA;
    if (KIND == MOE_PROBE_FP4)
      for (int c = 0; c < 2; ++c) {
        tc_cp_sf(tmem + 128 + c * 4, sdesc_sf(smem_u32(sfa + c * 512)));
        tc_cp_sf(tmem + 136 + c * 4, sdesc_sf(smem_u32(sfb + c * 512)));
      }
    const uint64_t t0 = globaltimer();
    const long long c0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t ad = sdesc_sw128(a_base + ks * 32), bd = sdesc_sw128(b_base + ks * 32);
        const uint32_t acc = (it > 0 || ks > 0);
        if (KIND == MOE_PROBE_FP8) {
          mma_f8f6f4(tmem, ad, bd, IDESC, acc);
        } else if (KIND == MOE_PROBE_FP4) {
          const int c = ks >> 1;
          const uint32_t sfid = (ks & 1) * 2;
          mma_mxf4(tmem, ad, bd, idesc_with_sf(IDESC, sfid, sfid), tmem + 128 + c * 4, tmem + 136 + c * 4, acc);
        } else {
          mma_bf16(tmem, ad, bd, IDESC, acc);
        }
      }
    }
    tc_commit(done);
    const bool ok = mbar_wait(done, 0, globaltimer() + timeout_ns, abort_flag);
    const uint64_t t1 = globaltimer();
    const long long c1 = clock64();
    g_probe[blockIdx.x][0] = ok ? t1 - t0 : 0ull;
    g_probe[blockIdx.x][1] = ok ? (unsigned long long)(c1 - c0) : 0ull;
    if (!ok) {   // let the tensor pipe drain before TMEM is released
      const uint64_t until = globaltimer() + 2000000ull;
      while (globaltimer() < until) { }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int KIND>
static cudaError_t probe_once(int grid, int iters, cudaStream_t st) {
  auto kern = k_tensor_probe<KIND>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
  if (e != cudaSuccess) return e;
  // an instruction takes well under 0.1 us; allow 1 us for each, plus 2 s
  const uint64_t timeout_ns = 2000000000ull + (uint64_t)iters * 4 * 1000ull;
  kern<<<grid, 128, kProbeSmem, st>>>(iters, timeout_ns);
  return cudaGetLastError();
}

// Runs a short warm-up, then the timed probe; *tflops = 2 * MACs of all CTAs
// over the slowest CTA's time, *mac_per_clk = the median CTA's MACs per SM
// clock.  Both 0 when a CTA's wait ran out.  Synchronizes the stream.
cudaError_t run_tensor_probe(int kind, int iters, cudaStream_t st, double* tflops, double* mac_per_clk) {
  int dev = 0, sms = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = sms < kProbeMaxCtas ? sms : kProbeMaxCtas;
  for (int pass = 0; pass < 2; ++pass) {
    const int n = pass == 0 ? (iters + 7) / 8 : iters;
    e = kind == MOE_PROBE_FP8 ? probe_once<MOE_PROBE_FP8>(grid, n, st)
      : kind == MOE_PROBE_FP4 ? probe_once<MOE_PROBE_FP4>(grid, n, st)
                              : probe_once<MOE_PROBE_BF16>(grid, n, st);
    if (e != cudaSuccess) return e;
  }
  unsigned long long host[kProbeMaxCtas][2];
  if ((e = cudaMemcpyFromSymbolAsync(host, g_probe, sizeof(unsigned long long) * 2 * grid, 0,
                                     cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return e;
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
  unsigned long long ns_max = 0;
  double rates[kProbeMaxCtas];
  bool ok = true;
  for (int i = 0; i < grid; ++i) {
    ok &= host[i][0] > 0 && host[i][1] > 0;
    if (host[i][0] > ns_max) ns_max = host[i][0];
    rates[i] = host[i][1] ? probe_macs_per_mma(kind) * 4.0 * iters / (double)host[i][1] : 0.0;
  }
  if (!ok) { *tflops = 0.0; *mac_per_clk = 0.0; return cudaSuccess; }
  for (int i = 1; i < grid; ++i)   // insertion sort: grid is the SM count
    for (int j = i; j > 0 && rates[j] < rates[j - 1]; --j) { const double t = rates[j]; rates[j] = rates[j - 1]; rates[j - 1] = t; }
  *mac_per_clk = rates[grid / 2];
  *tflops = 2.0 * probe_macs_per_mma(kind) * 4.0 * iters * grid / ((double)ns_max * 1e-9) / 1e12;
  return cudaSuccess;
}

}  // namespace moe
