// small.cu -- the whole MoE call in one launch for decode-sized batches
// (M <= 16 tokens, MXFP4 weights), where streaming the selected experts'
// weights from HBM is the work and every dependent memory round trip on the
// critical path shows.
//
// Grid: clusters of 4 CTAs, one CTA per SM, all co-resident.
//   prologue  every CTA routes all M tokens (a warp per token) and sorts the
//             pairs by expert in shared memory -- no routing kernel, no global
//             round trip; CTA 0 writes the debug taps.
//   GEMM1     cluster c takes (expert, n-tile) groups c, c + #clusters, ...; its
//             4 CTAs split K.  Weights by TMA; the token rows are quantized to
//             MXFP4 straight into the swizzled operand tile by a producer warp;
//             tcgen05 kind::mxf4, N = 16.  The split partials meet in rank 0's
//             epilogue through distributed shared memory (remote mbarrier
//             arrivals, reads in rank order), which applies SwiGLU, quantizes
//             mid once per (pair, 128) block to E4M3 with a power-of-two scale
//             ("glm53: FP8 mid hand-off", Modifications table row 1), stores
//             midq/midqs and publishes a per-(expert, n-tile) flag tagged with
//             the call's epoch ("glm53: FP8 mid hand-off": peers' sums tagged
//             with the launch's epoch).
//   GEMM2     cluster c takes h-tiles; rank r the experts r, r + 4, ... of the
//             selected list.  w2 tiles stream ahead by TMA; only the mid operand
//             waits for its expert's flags.  kind::mxf8f6f4 (E2M1 x E4M3).  The
//             epilogue accumulates w_j * y per token in registers (the combine,
//             "IQ2R: load GLM-5.3 packed MoE checkpoints": interleaved
//             down/reduction), the 4 ranks' sums meet in rank 0 through
//             distributed shared memory in rank order, and rank 0 writes bf16.
// Every result is produced in a fixed order: run-to-run identical.
#include <type_traits>

#include "codec.cuh"

namespace moe {

namespace small {

constexpr int NT = 16;           // token rows per MMA (N)
constexpr int CS = 4;            // CTAs per cluster
constexpr int STAGES = 4;
constexpr int A_BYTES = 16384;
constexpr int OFF_A1 = A_BYTES;
constexpr int OFF_B = 2 * A_BYTES;
constexpr int OFF_SFA = OFF_B + NT * 128;       // GEMM1: 4 chunks (gate c0,c1, up c0,c1); GEMM2: 1
constexpr int OFF_SFB = OFF_SFA + 4 * 512;      // 2 chunks (GEMM1), 1 (GEMM2)
constexpr int STAGE_BYTES = ((OFF_SFB + 2 * 512) + 1023) & ~1023;
constexpr int RED_FLOATS = 128 * 36;            // one reduction slot: 128 rows x (32 + 4 pad)
constexpr int NWARPS = 10;                      // 0 TMA, 1 MMA, 2-3 scales, 4-7 epilogue, 8-9 B operand
constexpr int THREADS = NWARPS * 32;
constexpr int MAX_P = 256;                      // M * topk
constexpr int MAX_J = 16;                       // I / 128
constexpr uint32_t IDESC1 = idesc_block_scaled(FMT4_E2M1, FMT4_E2M1, NT);
constexpr uint32_t IDESC2 = idesc_block_scaled(FMT8_E2M1, FMT8_E4M3, NT);
constexpr uint32_t TMEM_COLS = 128;             // acc buffers 2 x 32 columns, scales at 64..111
constexpr int SF_COL0 = 64;
constexpr int SF_SLOT = 24;
constexpr int KR_MAX = 8;                       // GEMM1 stages per rank (H <= 8192)
constexpr int XQ_ROW = KR_MAX * 128;            // packed E2M1 bytes of one token's K range
constexpr int XS_ROW = KR_MAX * 8;              // its E8M0 scales

struct Smem {
  int ids[MAX_P];
  float wts[MAX_P];
  int sorted_tok[MAX_P];     // token of each sorted pair
  float sorted_w[MAX_P];     // routing weight of each sorted pair
  int counts[kMaxE + 1];
  int offsets[kMaxE + 1];
  int dlist[kMaxE];          // selected experts, ascending
  int ndist;
  int epoch;
  int abort_flag;
  uint32_t tmem;
  uint64_t full[STAGES], empty[STAGES], accf[2], acce[2], red_full[2], red_free[2];
};
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 2 * RED_FLOATS * 4 + NT * 128 * 4 + NT * (XQ_ROW + XS_ROW) +
                           (int)sizeof(Smem) + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");

// The CTA's work, identical in every role: GEMM1 groups, then GEMM2 items.
struct Work {
  int ncl, cid, rank, kst1, kst2, J, HT, ngroups;
  __device__ int k0(int) const { return rank * kst1 / CS; }
  __device__ int k1(int) const { return (rank + 1) * kst1 / CS; }
};

__device__ __forceinline__ int htile_of(const Work& w, int n) {  // n-th h-tile of this cluster
  return n * w.ncl + (w.ncl - 1 - w.cid);                         // reverse order balances GEMM1
}

}  // namespace small

using namespace small;

__global__ void __launch_bounds__(THREADS, 1)
k_moe_small(const __grid_constant__ CUtensorMap tmW13, const __grid_constant__ CUtensorMap tmW2,
            const __grid_constant__ CUtensorMap tmMid, const SmallParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  float* red = reinterpret_cast<float*>(base + STAGES * STAGE_BYTES);        // [2][RED_FLOATS]
  float* epi = red + 2 * RED_FLOATS;                                          // [NT][128]
  uint8_t* xq_s = reinterpret_cast<uint8_t*>(epi + NT * 128);                 // [NT][XQ_ROW]
  uint8_t* xs_s = xq_s + NT * XQ_ROW;                                         // [NT][XS_ROW]
  Smem& S = *reinterpret_cast<Smem*>(xs_s + NT * XS_ROW);
  volatile int* abort_flag = &S.abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = p.M, E = p.E, k = p.topk, H = p.H, I = p.I, P = M * k;
  Work W;
  W.ncl = nclusters_x();
  W.cid = cluster_id_x();
  W.rank = cluster_ctarank();
  W.kst1 = H / 256;
  W.kst2 = I / 128;
  W.J = I / 128;
  W.HT = H / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&S.full[s], 3); mbar_init(&S.empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.accf[b], 1); mbar_init(&S.acce[b], 4);
      mbar_init(&S.red_full[b], CS - 1); mbar_init(&S.red_free[b], 1);
    }
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&tmW13); tma_prefetch_desc(&tmW2); tma_prefetch_desc(&tmMid); }
  if (warp == 1) { tmem_alloc(&S.tmem, TMEM_COLS); tmem_relinquish(); }
  // ---------------------------------------------------------------- routing, x quantization
  // Warps 0..min(M,10)-1 route a token each; the remaining warps (all warps,
  // after routing, when M >= 10) quantize every token's x over this rank's K
  // range into shared memory -- the GEMM1 operand rows are then copied from
  // there, with no global round trip per stage.
  {
    const int nrw = M < NWARPS ? M : NWARPS;
    for (int t = warp; t < M; t += NWARPS)
      route_token_warp(p.logits + (size_t)t * E, p.bias, E, k, p.routed_scale, &S.ids[t * k + lane],
                       &S.wts[t * k + lane]);
    const int kr0 = W.rank * W.kst1 / CS, kr = (W.rank + 1) * W.kst1 / CS - kr0;
    const int nblk = M * kr * 8;                      // 32-element blocks
    const int q0 = (nrw < NWARPS) ? nrw * 32 : 0, nq = THREADS - q0;
    for (int b = threadIdx.x - q0; b >= 0 && b < nblk; b += nq) {
      const int t = b / (kr * 8), lb = b % (kr * 8);
      const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)t * H + kr0 * 256 + lb * 32);
      uint4 u[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) u[c] = __ldg(src + c);
      float v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t w4[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[c * 8 + 2 * i] = __uint_as_float(w4[i] << 16);
          v[c * 8 + 2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
        }
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
      int code = 0;
      if (amax > 0.0f) code = max(0, min(254, floor_log2(amax) - 2 + 127));
      const float inv = exp2i(127 - code);
      uint32_t q[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(v[c * 8 + i], inv);
        q[c] = cvt_e2m1x8(f);
      }
      st_shared_v4(xq_s + t * XQ_ROW + lb * 16, q[0], q[1], q[2], q[3]);
      xs_s[t * XS_ROW + lb] = static_cast<uint8_t>(code);
    }
  }
  for (int e = threadIdx.x; e <= E; e += THREADS) S.counts[e] = 0;
  if (threadIdx.x == 0) S.epoch = __ldcg(p.sync) + 1;
  tc_fence_before();
  cluster_arrive_release();   // this CTA's barriers are initialized (waited for before the roles start)
  __syncthreads();
  for (int q = threadIdx.x; q < P; q += THREADS) atomicAdd(&S.counts[S.ids[q]], 1);
  __syncthreads();
  if (warp == 0) {  // exclusive scans: offsets and the list of selected experts
    const int per = (E + 31) / 32;
    int c[kMaxE / 32], nz[kMaxE / 32], s0 = 0, s1 = 0;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i) {
      const int e = lane * per + i;
      c[i] = (i < per && e < E) ? S.counts[e] : 0;
      nz[i] = c[i] > 0;
      s0 += c[i];
      s1 += nz[i];
    }
    int t0, t1;
    int o0 = warp_exclusive_scan(s0, &t0), o1 = warp_exclusive_scan(s1, &t1);
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i) {
      const int e = lane * per + i;
      if (i < per && e < E) {
        S.offsets[e] = o0;
        if (nz[i]) S.dlist[o1] = e;
      }
      o0 += c[i];
      o1 += nz[i];
    }
    if (lane == 0) { S.offsets[E] = t0; S.ndist = t1; }
  }
  __syncthreads();
  for (int q = threadIdx.x; q < P; q += THREADS) {  // stable position: ascending pair id inside an expert
    const int e = S.ids[q];
    int r = 0;
    for (int o = 0; o < q; ++o) r += (S.ids[o] == e);
    const int pos = S.offsets[e] + r;
    S.sorted_tok[pos] = q / k;
    S.sorted_w[pos] = S.wts[q];
    if (W.cid == 0 && W.rank == 0) { p.sorted_pairs[pos] = q; p.inv[q] = pos; }
  }
  if (W.cid == 0 && W.rank == 0) {  // debug taps
    for (int q = threadIdx.x; q < P; q += THREADS) { p.topk_ids[q] = S.ids[q]; p.topk_w[q] = S.wts[q]; }
    for (int e = threadIdx.x; e <= E; e += THREADS) {
      if (e < E) p.counts[e] = S.counts[e];
      p.offsets[e] = S.offsets[e];
    }
  }
  cluster_wait_acquire();   // every peer's barriers initialized before any remote arrival
  __syncthreads();
  tc_fence_after();         // the TMEM address written by warp 1
  W.ngroups = S.ndist * W.J;
  const int ndist = S.ndist, epoch = S.epoch;
  const uint32_t tmem = S.tmem;
  const uint64_t deadline = globaltimer() + p.timeout_ns;
  // items of GEMM2 for this CTA in one h-tile: experts rank, rank + CS, ...
  const int n_my2 = ndist > W.rank ? (ndist - W.rank + CS - 1) / CS : 0;
  int n_ht = 0;
  while (htile_of(W, n_ht) < W.HT) ++n_ht;

  auto fail = [&](int site, int a) {
    *abort_flag = 1;
    atomicOr(p.status, ST_TIMEOUT);
    atomicCAS(p.status + 2, 0,
              (int)(0x80000000u | (7u << 24) | ((unsigned)site << 20) | ((unsigned)min(a, 255) << 12) |
                    (blockIdx.x & 0xFFFu)));
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (weights)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int g = W.cid; g < W.ngroups && ok; g += W.ncl) {
        const int e = S.dlist[g / W.J], j = g % W.J;
        for (int kst = W.k0(g); kst < W.k1(g); ++kst) {
          if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { fail(1, kst); ok = false; break; }
          uint8_t* sb = stages + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&S.full[stage], 2 * A_BYTES);
          tma_load_3d(sb, &tmW13, &S.full[stage], kst * 128, j * 128, e);
          tma_load_3d(sb + OFF_A1, &tmW13, &S.full[stage], kst * 128, I + j * 128, e);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // this CTA's w2 tiles (and their scales) start moving into L2 while
      // GEMM1 drains and its results are published
      for (int n = 0; n < n_ht && ok; ++n)
        for (int it = 0; it < n_my2; ++it) {
          const size_t row0 = (size_t)S.dlist[W.rank + it * CS] * H + (size_t)htile_of(W, n) * 128;
          prefetch_l2_bulk(p.w2 + row0 * (I / 2), 64u * I);
          prefetch_l2_bulk(p.s2 + row0 * (I / 32), 4u * I);
        }
      for (int n = 0; n < n_ht && ok; ++n) {
        const int ht = htile_of(W, n);
        for (int it = 0; it < n_my2 && ok; ++it) {
          const int e = S.dlist[W.rank + it * CS];
          for (int kst = 0; kst < W.kst2; ++kst) {
            if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { fail(1, kst); ok = false; break; }
            uint8_t* sb = stages + stage * STAGE_BYTES;
            mbar_arrive_expect_tx(&S.full[stage], A_BYTES / 2);   // packed bytes of the unpacked 4-bit tile
            tma_load_3d(sb, &tmW2, &S.full[stage], kst * 128, ht * 128, e);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
      if (!ok) { const uint64_t until = globaltimer() + 2000000ull; while (globaltimer() < until) { } }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, it = 0, acc_n = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto run_stage = [&](bool g1, uint32_t d, bool first) -> bool {
        if (!mbar_wait(&S.full[stage], phase, deadline, abort_flag)) { fail(3, it); return false; }
        tc_fence_after();
        uint8_t* sb = stages + stage * STAGE_BYTES;
        const uint32_t sf0 = tmem + SF_COL0 + (it & 1) * SF_SLOT;
        const int nca = g1 ? 4 : 1, ncb = g1 ? 2 : 1;
        for (int c = 0; c < nca; ++c) tc_cp_sf(sf0 + c * 4, sdesc_sf(smem_u32(sb + OFF_SFA + c * 512)));
        for (int c = 0; c < ncb; ++c) tc_cp_sf(sf0 + 16 + c * 4, sdesc_sf(smem_u32(sb + OFF_SFB + c * 512)));
        const uint32_t a0 = smem_u32(sb), b0 = smem_u32(sb + OFF_B);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bd = sdesc_sw128(b0 + ks * 32);
          if (g1) {
            const int c = ks >> 1;
            const uint32_t id = idesc_with_sf(IDESC1, (ks & 1) * 2, (ks & 1) * 2);
            const uint32_t acc = (!first || ks > 0);
            mma_mxf4(d, sdesc_sw128(a0 + ks * 32), bd, id, sf0 + c * 4, sf0 + 16 + c * 4, acc);
            mma_mxf4(d + NT, sdesc_sw128(a0 + OFF_A1 + ks * 32), bd, id, sf0 + 8 + c * 4, sf0 + 16 + c * 4, acc);
          } else {
            const uint32_t id = idesc_with_sf(IDESC2, ks, ks);
            mma_mxf8f6f4(d, sdesc_sw128(a0 + ks * 32), bd, id, sf0, sf0 + 16, (!first || ks > 0));
          }
        }
        tc_commit(&S.empty[stage]);
        ++it;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
        return true;
      };
      auto acc_begin = [&]() -> uint32_t {
        const int b = acc_n & 1;
        if (!mbar_wait(&S.acce[b], ((acc_n >> 1) & 1) ^ 1, deadline, abort_flag)) { fail(2, acc_n); return 0xFFFFFFFFu; }
        tc_fence_after();
        return tmem + b * 32;
      };
      for (int g = W.cid; g < W.ngroups && ok; g += W.ncl) {
        if (W.k1(g) == W.k0(g)) continue;   // this rank has no K range: the epilogue writes zeros
        const uint32_t d = acc_begin();
        if (d == 0xFFFFFFFFu) { ok = false; break; }
        for (int kst = W.k0(g); kst < W.k1(g) && ok; ++kst) ok = run_stage(true, d, kst == W.k0(g));
        if (!ok) break;
        tc_commit(&S.accf[acc_n & 1]);
        ++acc_n;
      }
      for (int n = 0; n < n_ht && ok; ++n)
        for (int i2 = 0; i2 < n_my2 && ok; ++i2) {
          const uint32_t d = acc_begin();
          if (d == 0xFFFFFFFFu) { ok = false; break; }
          for (int kst = 0; kst < W.kst2 && ok; ++kst) ok = run_stage(false, d, kst == 0);
          if (!ok) break;
          tc_commit(&S.accf[acc_n & 1]);
          ++acc_n;
        }
      if (!ok) { tc_commit(&S.accf[0]); const uint64_t until = globaltimer() + 2000000ull; while (globaltimer() < until) { } }
    }
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------ weight scale factors
    // Stage s is always filled by warp 2 + (s & 1) (four stages: the parity of
    // the running stage count), so a warp only ever waits on its own stages and
    // its parity waits cannot alias.  GEMM1: a warp's words of a group are
    // loaded at once; GEMM2: the next item's words are loaded before the
    // current item is filled.
    const int sw = warp - 2;
    int stage = 0, it = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int g = W.cid; g < W.ngroups && ok; g += W.ncl) {
      const int e = S.dlist[g / W.J], j = g % W.J;
      const int k0 = W.k0(g), k1 = W.k1(g);
      uint32_t wa[KR_MAX / 2][2][2][4];
      const int i0 = (sw ^ it) & 1;   // this warp's first stage of the group: k0 + i0, then every other
#pragma unroll
      for (int b = 0; b < KR_MAX / 2; ++b) {
        const int kk = k0 + i0 + 2 * b;
        if (kk < k1) {
#pragma unroll
          for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const size_t row = (size_t)e * (2 * I) + (a2 ? I : 0) + j * 128 + lane + 32 * r;
                wa[b][a2][c][r] = __ldg(reinterpret_cast<const uint32_t*>(p.s13 + row * (H / 32) + kk * 8 + c * 4));
              }
        }
      }
      int mine = 0;
      for (int kst = k0; kst < k1; ++kst, ++it) {
        if ((it & 1) == sw) {
          if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { if (lane == 0) fail(5, kst); ok = false; break; }
          uint8_t* sb = stages + stage * STAGE_BYTES;
#pragma unroll
          for (int b = 0; b < KR_MAX / 2; ++b)
            if (b == mine)
#pragma unroll
              for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
                for (int c = 0; c < 2; ++c)
                  st_shared_v4(sb + OFF_SFA + (a2 * 2 + c) * 512 + lane * 16, wa[b][a2][c][0], wa[b][a2][c][1],
                               wa[b][a2][c][2], wa[b][a2][c][3]);
          ++mine;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.full[stage]);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    const int n_items = n_ht * n_my2;   // item i: h-tile i / n_my2, expert slot i % n_my2
    uint32_t wc[KR_MAX / 2][4], wn[KR_MAX / 2][4];   // this warp's words of the current / next item
    auto load_item = [&](int item, int it_first, uint32_t (&w)[KR_MAX / 2][4]) {
      const size_t row0 = (size_t)S.dlist[W.rank + (item % n_my2) * CS] * H + (size_t)htile_of(W, item / n_my2) * 128;
      const int i0 = (sw ^ it_first) & 1;
#pragma unroll
      for (int b = 0; b < KR_MAX / 2; ++b)
        if (i0 + 2 * b < W.kst2)
#pragma unroll
          for (int r = 0; r < 4; ++r)
            w[b][r] = __ldg(reinterpret_cast<const uint32_t*>(p.s2 + (row0 + lane + 32 * r) * (I / 32) +
                                                               (i0 + 2 * b) * 4));
    };
    if (ok && n_items > 0) load_item(0, it, wc);
    for (int item = 0; item < n_items && ok; ++item) {
      if (item + 1 < n_items) load_item(item + 1, it + W.kst2, wn);
      int mine = 0;
      for (int kst = 0; kst < W.kst2; ++kst, ++it) {
        if ((it & 1) == sw) {
          if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { if (lane == 0) fail(5, kst); ok = false; break; }
          uint8_t* sb = stages + stage * STAGE_BYTES;
#pragma unroll
          for (int b = 0; b < KR_MAX / 2; ++b)
            if (b == mine) st_shared_v4(sb + OFF_SFA + lane * 16, wc[b][0], wc[b][1], wc[b][2], wc[b][3]);
          ++mine;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.full[stage]);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
#pragma unroll
      for (int b = 0; b < KR_MAX / 2; ++b)
#pragma unroll
        for (int r = 0; r < 4; ++r) wc[b][r] = wn[b][r];
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ B operand (tokens / mid)
    // GEMM1: stage s is filled by warp 8 + (s & 1), rows copied from the
    // quantized tokens in shared memory.  GEMM2: once both warps are past
    // GEMM1 (so every stage has been filled for the last time by its GEMM1
    // owner), one thread of warp 8 fills every stage: it waits for the
    // (expert, k-block) mid flag of the call, then loads the mid rows by TMA and
    // their scale-factor rows, stored in MMA layout by the publisher, by bulk copy.
    const int bw = warp - 8;
    int stage = 0, it = 0;
    uint32_t phase = 0;
    bool ok = true;
    const int m = lane >> 1, half = lane & 1;   // GEMM1: row m, 64-byte half of the 128-byte stage row
    for (int g = W.cid; g < W.ngroups && ok; g += W.ncl) {
      const int e = S.dlist[g / W.J];
      const int cnt = S.counts[e], off = S.offsets[e];
      const int t = m < cnt ? S.sorted_tok[off + m] : -1;
      for (int kst = W.k0(g); kst < W.k1(g); ++kst, ++it) {
        if ((it & 1) == bw) {
          const int ls = kst - W.k0(g);   // stage inside this rank's quantized range
          uint4 q[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
          uint32_t sfw = 0;
          if (t >= 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              q[c] = *reinterpret_cast<const uint4*>(xq_s + t * XQ_ROW + ls * 128 + half * 64 + c * 16);
            sfw = *reinterpret_cast<const uint32_t*>(xs_s + t * XS_ROW + ls * 8 + half * 4);
          }
          if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { if (lane == 0) fail(6, kst); ok = false; break; }
          uint8_t* sb = stages + stage * STAGE_BYTES;
#pragma unroll
          for (int c = 0; c < 4; ++c) {   // 16-byte chunks of the row, 128-byte swizzle
            const int ck = half * 4 + c;
            st_shared_v4(sb + OFF_B + m * 128 + ((ck ^ (m & 7)) * 16), q[c].x, q[c].y, q[c].z, q[c].w);
          }
          *reinterpret_cast<uint32_t*>(sb + OFF_SFB + half * 512 + m * 16) = sfw;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.full[stage]);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    named_bar_sync(2, 64);   // both B warps done with GEMM1 (a failed warp arrives too)
    if (bw == 0 && lane == 0 && ok) {
      const int n_items = n_ht * n_my2;
      for (int item = 0; item < n_items && ok; ++item) {
        const int e = S.dlist[W.rank + (item % n_my2) * CS];
        const int off = S.offsets[e];
        for (int kst = 0; kst < W.kst2; ++kst) {
          uint32_t spins = 0;
          while (ld_acquire_gpu(p.flags + e * MAX_J + kst) != epoch) {
            if ((++spins & 63u) == 0 && (*abort_flag || globaltimer() > deadline)) { fail(7, e); ok = false; break; }
          }
          if (!ok) break;
          fence_proxy_async_global();
          if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { fail(6, kst); ok = false; break; }
          uint8_t* sb = stages + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&S.full[stage], NT * 128 + NT * 16);
          tma_load_2d(sb + OFF_B, &tmMid, &S.full[stage], kst * 128, off);
          bulk_load(sb + OFF_SFB, p.midsf + ((size_t)e * W.kst2 + kst) * 64, NT * 16, &S.full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) { const uint64_t until = globaltimer() + 2000000ull; while (globaltimer() < until) { } }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (warps 4..7)
    const int ew = warp - 4, row = 32 * ew + lane;   // TMEM lane quarter = warp % 4
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * ew) << 16);
    const uint32_t red_s = smem_u32(red);
    int acc_n = 0, red_n = 0;
    bool ok = true;
    // cross-rank reduction of `vals` (n floats per row) in rank order; rank 0
    // gets the sum.  Rank 0 issues all loads of a batch of peers before adding,
    // so a batch costs one distributed-shared-memory round trip.
    auto reduce = [&](float* vals, auto n_const) -> bool {
      constexpr int n = decltype(n_const)::value;
      constexpr int RB = n <= 16 ? CS - 1 : 1;   // peers per batch
      const int slot = red_n & 1;
      const uint32_t par = (red_n >> 1) & 1;
      ++red_n;
      if (W.rank != 0) {
        if (!mbar_wait_cluster(&S.red_free[slot], par ^ 1, deadline, abort_flag)) { fail(8, 0); return false; }
        float* dst = red + slot * RED_FLOATS + row * 36;
#pragma unroll
        for (int i = 0; i < n; i += 4)
          *reinterpret_cast<float4*>(dst + i) = make_float4(vals[i], vals[i + 1], vals[i + 2], vals[i + 3]);
        named_bar_sync(1, 128);
        if (ew == 0 && lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.red_full[slot]), 0));
        return true;
      }
      if (!mbar_wait_cluster(&S.red_full[slot], par, deadline, abort_flag)) { fail(9, 0); return false; }
      const uint32_t mine = red_s + (slot * RED_FLOATS + row * 36) * 4;
#pragma unroll
      for (int r0 = 1; r0 < CS; r0 += RB) {
        float4 t[RB][n / 4];
#pragma unroll
        for (int rr = 0; rr < RB; ++rr) {
          const uint32_t src = mapa_shared(mine, r0 + rr);
#pragma unroll
          for (int i = 0; i < n / 4; ++i) t[rr][i] = ld_shared_cluster_f4(src + i * 16);
        }
#pragma unroll
        for (int rr = 0; rr < RB; ++rr)
#pragma unroll
          for (int i = 0; i < n / 4; ++i) {
            vals[4 * i] += t[rr][i].x; vals[4 * i + 1] += t[rr][i].y;
            vals[4 * i + 2] += t[rr][i].z; vals[4 * i + 3] += t[rr][i].w;
          }
      }
      named_bar_sync(1, 128);   // all rows read before the peers may overwrite
      if (ew == 0 && lane < CS && lane > 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.red_free[slot]), lane));
      return true;
    };
    for (int g = W.cid; g < W.ngroups && ok; g += W.ncl) {
      const int e = S.dlist[g / W.J], j = g % W.J;
      float v[32];   // gate columns 0..15, up columns 16..31 of this row
      if (W.k1(g) > W.k0(g)) {
        const int b = acc_n & 1;
        if (!mbar_wait(&S.accf[b], (acc_n >> 1) & 1, deadline, abort_flag)) { fail(10, 0); ok = false; break; }
        tc_fence_after();
        float gg[16], uu[16];
        tmem_ld16(tl + b * 32, gg);
        tmem_ld16(tl + b * 32 + NT, uu);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acce[b]);
        ++acc_n;
#pragma unroll
        for (int i = 0; i < 16; ++i) { v[i] = gg[i]; v[16 + i] = uu[i]; }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
      }
      if (!reduce(v, std::integral_constant<int, 32>())) { ok = false; break; }
      if (W.rank != 0) continue;
      const int cnt = S.counts[e], off = S.offsets[e];
#pragma unroll
      for (int c = 0; c < NT; ++c) epi[c * 128 + row] = v[c] / (1.0f + expf(-v[c])) * v[16 + c];
      named_bar_sync(1, 128);
      for (int c = ew; c < cnt; c += 4) {   // mid quantized once per (pair, 128-block)
        const float4 q4 = reinterpret_cast<const float4*>(epi + c * 128)[lane];
        float amax = fmaxf(fmaxf(fabsf(q4.x), fabsf(q4.y)), fmaxf(fabsf(q4.z), fabsf(q4.w)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const int ke = pow2_e4m3_exp(amax);
        const float inv = exp2i(-ke);
        const size_t r = (size_t)(off + c);
        reinterpret_cast<uint32_t*>(p.midq + r * I + j * 128)[lane] =
            cvt_e4m3x4(q4.x * inv, q4.y * inv, q4.z * inv, q4.w * inv);
        if (lane == 0) {
          p.midqs[r * (I / 128) + j] = exp2i(ke);
          p.midsf[((size_t)e * W.J + j) * 64 + c * 4] = rep4((uint32_t)(ke + 127));   // B scale row c, E8M0
        }
      }
      __threadfence();
      named_bar_sync(1, 128);
      if (ew == 0 && lane == 0) st_release_gpu(p.flags + e * MAX_J + j, epoch);
    }
    for (int n = 0; n < n_ht && ok; ++n) {
      const int ht = htile_of(W, n);
      float acc[NT];
#pragma unroll
      for (int i = 0; i < NT; ++i) acc[i] = 0.0f;
      for (int i2 = 0; i2 < n_my2 && ok; ++i2) {
        const int e = S.dlist[W.rank + i2 * CS];
        const int cnt = S.counts[e], off = S.offsets[e];
        const int b = acc_n & 1;
        if (!mbar_wait(&S.accf[b], (acc_n >> 1) & 1, deadline, abort_flag)) { fail(10, 1); ok = false; break; }
        tc_fence_after();
        float y[16];
        tmem_ld16(tl + b * 32, y);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acce[b]);
        ++acc_n;
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          if (c < cnt) {
            const int t = S.sorted_tok[off + c];
            const float w = S.sorted_w[off + c];
#pragma unroll
            for (int tt = 0; tt < NT; ++tt)
              if (tt == t) acc[tt] = fmaf(w, y[c], acc[tt]);
          }
        }
      }
      if (!ok) break;
      if (!reduce(acc, std::integral_constant<int, NT>())) { ok = false; break; }
      if (W.rank == 0) {
        for (int t = 0; t < M; ++t) {
          const uint32_t b2 = pack_bf16x2(acc[t], 0.0f) & 0xFFFFu;
          p.out[(size_t)t * H + ht * 128 + row] = static_cast<uint16_t>(b2);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  cluster_sync_all();   // no CTA leaves while a peer may still read its shared memory
  if (threadIdx.x == 0) {
    const int old = atomicAdd(p.sync + 1, 1);
    if (old == (int)gridDim.x - 1) {     // last CTA of the call: advance the epoch
      p.sync[1] = 0;
      __threadfence();
      st_release_gpu(p.sync, epoch);
    }
  }
}

// ---------------------------------------------------------------------------
int small_max_clusters(int dev) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    cudaFuncSetAttribute(k_moe_small, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CS);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_moe_small, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = -1;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

cudaError_t launch_small(const CUtensorMap& w13, const CUtensorMap& w2, const CUtensorMap& mid,
                         const SmallParams& p, int nclusters, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nclusters * CS);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_moe_small, w13, w2, mid, p);
}

}  // namespace moe
