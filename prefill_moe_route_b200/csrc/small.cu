// small.cu -- the whole MoE call in one launch for decode-sized batches
// (M <= 16 tokens, MXFP4 weights), where streaming the selected experts'
// weights from HBM is the work and every dependent memory round trip on the
// critical path shows.
//
// Grid: clusters of CS = 4 CTAs, one CTA per SM, all co-resident.
//   prologue  every CTA routes all M tokens (a warp per token), sorts the
//             pairs by expert in shared memory and quantizes the tokens to
//             MXFP4 over its rank's K range straight into a GEMM1 operand
//             that stays in shared memory for the whole call (all M tokens are
//             the N = 16 columns of every GEMM1 tile); CTA 0 writes the taps.
//   GEMM1     cluster c takes (expert, n-tile) groups c, c + #clusters, ...; its
//             CS CTAs split K.  One thread streams the gate and up tiles by TMA
//             and their scale blocks (stored in the tensor cores' order) by
//             bulk copy; tcgen05 kind::mxf4.  The split partials meet in rank
//             0's epilogue through distributed shared memory (remote mbarrier
//             arrivals, reads in rank order), which applies SwiGLU, quantizes
//             mid once per (pair, 128) block to E4M3 with a power-of-two scale
//             ("glm53: FP8 mid hand-off", Modifications table row 1), stores
//             midq/midqs plus the scale rows in the MMA's order, and publishes
//             a per-(expert, k-block) flag tagged with the call's epoch
//             ("glm53: FP8 mid hand-off": peers' sums tagged with the launch's
//             epoch).
//   GEMM2     cluster c takes an h-tile, and half of the experts of one more
//             when there are more h-tiles than clusters (the two halves'
//             sums meet in the owner, in order, through global memory);
//             rank r the experts r, r + CS, ... of the selected list.  w2 tiles and scales stream ahead by TMA; one
//             warp polls the mid flags and moves mid, kept as 16 token rows
//             per expert, from L2 into the stages through registers.
//             kind::mxf8f6f4 (E2M1 x E4M3), two k-steps per stage;
//             accumulator column t is token t.  The epilogue accumulates w_j * y per token (the
//             combine, "IQ2R: load GLM-5.3 packed MoE checkpoints":
//             interleaved down/reduction), the ranks' sums meet in rank 0
//             through distributed shared memory in rank order, and rank 0
//             writes bf16.
// Every result is produced in a fixed order: run-to-run identical.
#include <type_traits>

#include "codec.cuh"

namespace moe {

namespace small {

constexpr int NT = 16;           // MMA N: the token columns of both GEMMs
constexpr int CS = 4;            // CTAs per cluster
constexpr int STAGES = 4;
constexpr int A_TILE = 16384;    // one 128 x 128-byte operand tile in shared memory
// stage layout.  GEMM1: gate tile, up tile, 4 scale blocks (gate c0 c1, up c0 c1).
// GEMM2: up to KS2 k-steps of w2, each a tile and a scale block (mid is held per expert).
constexpr int G1_SFA = 2 * A_TILE;
constexpr int KS2 = 2;
constexpr int G2_SFA = KS2 * A_TILE;            // + k * 512
constexpr int STAGE_BYTES = G1_SFA + 2048;
static_assert(STAGE_BYTES % 1024 == 0 && G2_SFA + KS2 * 512 <= STAGE_BYTES, "stage layout");
constexpr int KR_MAX = 8;                   // GEMM1 stages per rank (H <= 256 * CS * KR_MAX)
constexpr int XB_BYTES = KR_MAX * NT * 128; // persistent GEMM1 token operand: one 16 x 128-byte tile per stage
constexpr int MID_BYTES = 32 * 1024;        // the same space, extended: GEMM2's mid buffers after GEMM1
constexpr int MAX_MIDBUF = 8;
constexpr int XSF_PITCH = 256;              // its scale blocks: rows 0..15 are the first 256 bytes of a block
constexpr int XSF_BYTES = KR_MAX * 2 * XSF_PITCH + 256;   // + the last block's unread second half
constexpr int RED_FLOATS = 128 * 32;        // one reduction slot: 128 rows x 32, float4s XOR-swizzled by row
constexpr int NWARPS = 8;                   // 0 TMA, 1 MMA, 2 mid operand, 3 set-up help, 4-7 epilogue
constexpr int THREADS = NWARPS * 32;
constexpr int MAX_P = 256;                  // M * topk
constexpr int MAX_J = 16;                   // I / 128
constexpr uint32_t IDESC1 = idesc_block_scaled(FMT4_E2M1, FMT4_E2M1, NT);
constexpr uint32_t IDESC2 = idesc_block_scaled(FMT8_E2M1, FMT8_E4M3, NT);
constexpr int NACC = 4;                     // TMEM accumulator buffers
constexpr uint32_t TMEM_COLS = 256;         // acc buffers 4 x 32 columns, scales at 128..239
constexpr int SF_COL0 = NACC * 32;          // per-stage weight scales, 2 slots
constexpr int SF_SLOT = 24;
constexpr int XSFB_COL = SF_COL0 + 2 * SF_SLOT;   // token / mid scale blocks, 16 x 4 columns (to 240)

// Prologue-only arrays, kept in the reduction buffers (first written after the prologue).
struct Pro {
  int ids[MAX_P];
  float wts[MAX_P];
  float sorted_w[MAX_P];     // routing weight of each sorted pair
};
static_assert(sizeof(Pro) <= 2 * RED_FLOATS * 4, "prologue arrays");

struct Smem {
  uint8_t sorted_tok[MAX_P]; // token of each sorted pair
  int counts[kMaxE + 1];
  int offsets[kMaxE + 1];
  uint16_t dlist[kMaxE];     // selected experts, ascending
  alignas(16) float wtok[(MAX_P + CS - 1) / CS][NT];  // GEMM2 expert slot i2 of this rank: weight of token t (0: not routed)
  int ndist;
  int epoch;
  int abort_flag;
  uint32_t tmem;
  uint64_t full[STAGES], empty[STAGES], accf[NACC], acce[NACC], red_full[2], red_free[2], g1done;
  uint64_t midfull[MAX_MIDBUF], midempty[MAX_MIDBUF];   // GEMM2's mid buffers (in the token operand's space)
  uint64_t epibar;           // the 4 epilogue warps' barrier (bounded, unlike bar.sync)
  int xok;                   // the owner's wait for its partner half succeeded
};
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + MID_BYTES + XSF_BYTES + 2 * RED_FLOATS * 4 + NT * 128 * 4 +
                           (int)sizeof(Smem) + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");

// The CTA's work, identical in every role: GEMM1 groups, then GEMM2 items.
struct Work {
  int ncl, cid, rank, kst1, kst2, J, HT, ngroups;
  int k0, k1;                 // this rank's GEMM1 stages (of 256 K elements)
};

// GEMM2 units of a cluster: h-tile ht[u] with all of the selected experts
// (half 0), or one half of them: an h-tile beyond one per cluster is split
// between two clusters, the owner (half 1, experts of each rank's first
// half) adding its partner's partial (half 2, the rest) in that order.  When
// there are too many h-tiles for halves, a cluster takes two whole ones.
struct Units {
  int n, ht[2], half[2];
};
__device__ __forceinline__ Units units_of(const Work& w) {
  Units u;
  const int HT = w.HT, ncl = w.ncl, c = w.ncl - 1 - w.cid;   // reverse order: clusters with fewer GEMM1 groups first
  u.n = 0;
  if (c < HT) { u.ht[0] = c; u.half[0] = 0; u.n = 1; }
  const int extra = HT - ncl;
  if (extra > 0 && 2 * extra <= ncl) {
    if (c < 2 * extra) { u.ht[1] = ncl + c / 2; u.half[1] = 1 + (c & 1); u.n = 2; }
  } else if (extra > 0 && ncl + c < HT) {
    u.ht[1] = ncl + c; u.half[1] = 0; u.n = 2;
  }
  return u;
}
// whether unit u takes this rank's expert slot i2 (of n_my2)
__device__ __forceinline__ bool unit_has(const Units& U, int u, int i2, int n_my2) {
  const int h = U.half[u], split = (n_my2 + 1) / 2;
  return h == 0 || (h == 1 ? i2 < split : i2 >= split);
}

}  // namespace small

using namespace small;

// NTOK: the token columns an epilogue carries (M rounded up to 4), so the
// cross-rank reductions move 2 NTOK (GEMM1) or NTOK (GEMM2) floats per row.
template <int NTOK>
__global__ void __launch_bounds__(THREADS, 1)
k_moe_small(const __grid_constant__ CUtensorMap tmW13, const __grid_constant__ CUtensorMap tmW2,
            const __grid_constant__ CUtensorMap tmMid, const SmallParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = base;
  uint8_t* xb = base + STAGES * STAGE_BYTES;   // GEMM1: [KR_MAX][16][128] swizzled tokens; GEMM2: mid buffers
  uint8_t* xsf = xb + MID_BYTES;               // their scale blocks, 256 B pitch
  float* red = reinterpret_cast<float*>(xsf + XSF_BYTES);                      // [2][RED_FLOATS]
  float* epi = red + 2 * RED_FLOATS;                                           // [NT][128]
  Smem& S = *reinterpret_cast<Smem*>(epi + NT * 128);
  Pro& PR = *reinterpret_cast<Pro*>(red);
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
  W.k0 = W.rank * W.kst1 / CS;
  W.k1 = (W.rank + 1) * W.kst1 / CS;
  const int KR = W.k1 - W.k0;
  const int prev_epoch = threadIdx.x == 0 ? __ldcg(p.sync) : 0;   // in flight while routing runs

  // set-up by the last warp, which routes a token only when M = 8 or more
  if (threadIdx.x == THREADS - 32) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&S.full[s], 2); mbar_init(&S.empty[s], 1); }
    for (int b = 0; b < NACC; ++b) { mbar_init(&S.accf[b], 1); mbar_init(&S.acce[b], 4); }
    for (int b = 0; b < 2; ++b) { mbar_init(&S.red_full[b], CS - 1); mbar_init(&S.red_free[b], 1); }
    mbar_init(&S.g1done, 1);
    for (int b = 0; b < MAX_MIDBUF; ++b) { mbar_init(&S.midfull[b], 1); mbar_init(&S.midempty[b], 1); }
    mbar_init(&S.epibar, 128);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == THREADS - 31) { tma_prefetch_desc(&tmW13); tma_prefetch_desc(&tmW2); }
  if (warp == NWARPS - 1) { tmem_alloc(&S.tmem, TMEM_COLS); tmem_relinquish(); }
  // ---------------------------------------------------------------- routing, x quantization
  // Warps 0..min(M,8)-1 route a token each (two when M > 8); the other warps,
  // then all of them, quantize the 16 operand rows over this rank's K range:
  // token t < M from x, rows M..15 zero.
  {
    const int nrw = M < NWARPS ? M : NWARPS;
    for (int t = warp; t < M; t += NWARPS) {   // scratch: this warp's 4 KB of the idle stage ring
      if (p.ids_in)
        take_routed_token(p.ids_in + (size_t)t * k, p.w_in + (size_t)t * k, E, k, &PR.ids[t * k + lane],
                          &PR.wts[t * k + lane], p.status);
      else
        route_token_warp(p.logits + (size_t)t * E, p.bias, E, k, p.routed_scale, &PR.ids[t * k + lane],
                         &PR.wts[t * k + lane], reinterpret_cast<uint32_t*>(stages) + warp * 2 * kMaxE);
    }
    const int nblk = NT * KR * 8;                     // 32-element blocks
    const int q0 = (nrw < NWARPS) ? nrw * 32 : 0, nq = THREADS - q0;
    for (int b = threadIdx.x - q0; b >= 0 && b < nblk; b += nq) {
      const int t = b / (KR * 8), lb = b % (KR * 8), ls = lb >> 3, j8 = lb & 7;
      uint32_t q[4] = {0u, 0u, 0u, 0u};
      int code = 0;
      if (t < M) {
        const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)t * H + W.k0 * 256 + lb * 32);
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
        if (amax > 0.0f) code = max(0, min(254, floor_log2(amax) - 2 + 127));
        const float inv = exp2i(127 - code);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(v[c * 8 + i], inv);
          q[c] = cvt_e2m1x8(f);
        }
      }
      // 16-byte chunk j8 of row t in the 128-byte swizzled tile of stage ls
      st_shared_v4(xb + ls * (NT * 128) + t * 128 + ((j8 ^ (t & 7)) * 16), q[0], q[1], q[2], q[3]);
      // scale byte (j8 % 4) of row t in block (ls, j8 / 4): byte 16 t + j8 % 4
      xsf[(ls * 2 + (j8 >> 2)) * XSF_PITCH + t * 16 + (j8 & 3)] = static_cast<uint8_t>(code);
    }
    fence_proxy_async_smem();   // the operand is read by the tensor cores
  }
  for (int e = threadIdx.x; e <= E; e += THREADS) S.counts[e] = 0;
  if (threadIdx.x == 0) S.epoch = prev_epoch + 1;
  tc_fence_before();
  cluster_arrive_release();   // this CTA's barriers are initialized (waited for before the roles start)
  __syncthreads();
  for (int q = threadIdx.x; q < P; q += THREADS) atomicAdd(&S.counts[PR.ids[q]], 1);
  __syncthreads();
  if (warp == 0) {  // exclusive scans: offsets and the list of selected experts (lane: `per` experts)
    const int per = (E + 31) / 32, e0 = lane * per, e1 = min(E, e0 + per);
    int s0 = 0, s1 = 0;
#pragma unroll 1
    for (int e = e0; e < e1; ++e) { const int c = S.counts[e]; s0 += c; s1 += c > 0; }
    int t0, t1;
    int o0 = warp_exclusive_scan(s0, &t0), o1 = warp_exclusive_scan(s1, &t1);
#pragma unroll 1
    for (int e = e0; e < e1; ++e) {
      const int c = S.counts[e];
      S.offsets[e] = o0;
      if (c > 0) S.dlist[o1++] = static_cast<uint16_t>(e);
      o0 += c;
    }
    if (lane == 0) { S.offsets[E] = t0; S.ndist = t1; }
  }
  __syncthreads();
  for (int q = threadIdx.x; q < P; q += THREADS) {  // stable position: ascending pair id inside an expert
    const int e = PR.ids[q];
    int r = 0;
    for (int o = 0; o < q; ++o) r += (PR.ids[o] == e);
    const int pos = S.offsets[e] + r;
    S.sorted_tok[pos] = static_cast<uint8_t>(q / k);
    PR.sorted_w[pos] = PR.wts[q];
    if (W.cid == 0 && W.rank == 0) { p.sorted_pairs[pos] = q; p.inv[q] = pos; }
  }
  __syncthreads();
  {  // routing weight of each token for this rank's GEMM2 experts
    const int nd = S.ndist, nm = nd > W.rank ? (nd - W.rank + CS - 1) / CS : 0;
    for (int i = threadIdx.x; i < nm * NT; i += THREADS) {
      const int i2 = i / NT, t = i % NT, e = S.dlist[W.rank + i2 * CS];
      const int off = S.offsets[e], cnt = S.counts[e];
      float w = 0.0f;
      for (int c = 0; c < cnt; ++c)   // a token that names an expert twice counts twice
        if (S.sorted_tok[off + c] == t) w += PR.sorted_w[off + c];
      S.wtok[i2][t] = w;
    }
  }
  if (W.cid == 0 && W.rank == 0) {  // debug taps
    for (int q = threadIdx.x; q < P; q += THREADS) { p.topk_ids[q] = PR.ids[q]; p.topk_w[q] = PR.wts[q]; }
    for (int e = threadIdx.x; e <= E; e += THREADS) {
      if (e < E) p.counts[e] = S.counts[e];
      p.offsets[e] = S.offsets[e];
    }
  }
  cluster_wait_acquire();   // every peer's barriers initialized before any remote arrival
  __syncthreads();
  tc_fence_after();         // the TMEM address written by the last warp
  W.ngroups = S.ndist * W.J;
  const int ndist = S.ndist, epoch = S.epoch;
  const uint32_t tmem = S.tmem;
  const uint64_t deadline = globaltimer() + p.timeout_ns;
  // GEMM2 units (h-tiles or halves of them) of this cluster; the items of
  // this CTA are its experts rank, rank + CS, ... on each unit that takes them
  const Units U = units_of(W);   // the launch requires H / 128 <= 2 * #clusters
  const int n_my2 = (U.n > 0 && ndist > W.rank) ? (ndist - W.rank + CS - 1) / CS : 0;
  // GEMM2 items run expert-major: expert slot i2, then its units.
  // Each expert's mid (kst2 tiles of 16 x 128 bytes + scale rows) is loaded
  // once into one of `nbuf` buffers in the GEMM1 token operand's space.
  const int nbuf = min(MAX_MIDBUF, min(MID_BYTES / (W.kst2 * NT * 128), 16 / W.kst2));

  auto fail = [&](int site, int a) {
    *abort_flag = 1;
    atomicOr(p.status, ST_TIMEOUT);
    atomicCAS(p.status + 2, 0,
              (int)(0x80000000u | (7u << 24) | ((unsigned)site << 20) | ((unsigned)min(a, 255) << 12) |
                    (blockIdx.x & 0xFFFu)));
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (weights and their scales)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const size_t sblk13 = (size_t)(H / 128) * 512;   // bytes of one 128-row tile's scale blocks (w13)
      for (int g = W.cid; g < W.ngroups && ok; g += W.ncl) {
        const int e = S.dlist[g / W.J], j = g % W.J;
        const uint8_t* sg = p.s13 + ((size_t)e * (2 * I / 128) + j) * sblk13;           // gate tile's blocks
        const uint8_t* su = p.s13 + ((size_t)e * (2 * I / 128) + I / 128 + j) * sblk13; // up tile's blocks
        for (int kst = W.k0; kst < W.k1; ++kst) {
          if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { fail(1, kst); ok = false; break; }
          uint8_t* sb = stages + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&S.full[stage], 2 * A_TILE + 2048);
          mbar_arrive(&S.full[stage]);   // GEMM1 stages have no second producer
          tma_load_3d(sb, &tmW13, &S.full[stage], kst * 128, j * 128, e);
          tma_load_3d(sb + A_TILE, &tmW13, &S.full[stage], kst * 128, I + j * 128, e);
          bulk_load(sb + G1_SFA, sg + (size_t)kst * 1024, 1024, &S.full[stage]);
          bulk_load(sb + G1_SFA + 1024, su + (size_t)kst * 1024, 1024, &S.full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      for (int i2 = 0; i2 < n_my2 && ok; ++i2) {
        const int e = S.dlist[W.rank + i2 * CS];
        for (int u = 0; u < U.n && ok; ++u) {
          if (!unit_has(U, u, i2, n_my2)) continue;
          const int ht = U.ht[u];
          const uint8_t* s2b = p.s2 + ((size_t)e * W.HT + ht) * (size_t)(I / 128) * 512;
          for (int k0 = 0; k0 < W.kst2; k0 += KS2) {
            const int nk = min(KS2, W.kst2 - k0);
            if (!mbar_wait(&S.empty[stage], phase ^ 1, deadline, abort_flag)) { fail(1, k0); ok = false; break; }
            uint8_t* sb = stages + stage * STAGE_BYTES;
            mbar_arrive_expect_tx(&S.full[stage], nk * (A_TILE / 2 + 512));   // 4-bit tiles land unpacked
            mbar_arrive(&S.full[stage]);   // the stage's only producer
            for (int kk = 0; kk < nk; ++kk)
              tma_load_3d(sb + kk * A_TILE, &tmW2, &S.full[stage], (k0 + kk) * 128, ht * 128, e);
            bulk_load(sb + G2_SFA, s2b + (size_t)k0 * 512, nk * 512, &S.full[stage]);
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
      // A full stage holds only TMA / bulk-copy data (async proxy, like the
      // MMA's reads), ordered by the barrier's transaction count: no tcgen05
      // fence, so the tensor pipe keeps running across stages.
      auto wait_full = [&]() -> bool {
        if (!mbar_wait(&S.full[stage], phase, deadline, abort_flag)) { fail(3, it); return false; }
        return true;
      };
      auto release = [&]() {
        tc_commit(&S.empty[stage]);
        ++it;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      };
      auto acc_begin = [&]() -> uint32_t {
        const int b = acc_n % NACC;
        if (!mbar_wait(&S.acce[b], ((acc_n / NACC) & 1) ^ 1, deadline, abort_flag)) { fail(2, acc_n); return 0xFFFFFFFFu; }
        tc_fence_after();
        return tmem + b * 32;
      };
      const uint32_t xb_s = smem_u32(xb), xsf_s = smem_u32(xsf);
      for (int i = 0; i < 2 * KR; ++i)   // the token operand's scale blocks stay in TMEM for GEMM1
        tc_cp_sf(tmem + XSFB_COL + i * 4, sdesc_sf(xsf_s + i * XSF_PITCH));
      for (int g = W.cid; g < W.ngroups && ok && KR > 0; g += W.ncl) {
        const uint32_t d = acc_begin();
        if (d == 0xFFFFFFFFu) { ok = false; break; }
        for (int kst = W.k0; kst < W.k1 && ok; ++kst) {
          if (!(ok = wait_full())) break;
          const uint32_t sb = smem_u32(stages + stage * STAGE_BYTES);
          const uint32_t sf0 = tmem + SF_COL0 + (it & 1) * SF_SLOT;
          const int ls = kst - W.k0;
          for (int c = 0; c < 4; ++c) tc_cp_sf(sf0 + c * 4, sdesc_sf(sb + G1_SFA + c * 512));
          const uint32_t b0 = xb_s + ls * (NT * 128), xs0 = tmem + XSFB_COL + ls * 8;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bd = sdesc_sw128(b0 + ks * 32);
            const int c = ks >> 1;
            const uint32_t id = idesc_with_sf(IDESC1, (ks & 1) * 2, (ks & 1) * 2);
            const uint32_t acc = (kst > W.k0 || ks > 0);
            mma_mxf4(d, sdesc_sw128(sb + ks * 32), bd, id, sf0 + c * 4, xs0 + c * 4, acc);
            mma_mxf4(d + NT, sdesc_sw128(sb + A_TILE + ks * 32), bd, id, sf0 + 8 + c * 4, xs0 + c * 4, acc);
          }
          release();
        }
        if (!ok) break;
        tc_commit(&S.accf[acc_n % NACC]);
        ++acc_n;
      }
      tc_commit(&S.g1done);   // every GEMM1 stage consumed: the mid-operand warp may take over
      for (int i2 = 0; i2 < n_my2 && ok; ++i2) {
        const int buf = i2 % nbuf, use = i2 / nbuf;
        if (!mbar_wait(&S.midfull[buf], use & 1, deadline, abort_flag)) { fail(11, i2); ok = false; break; }
        const uint32_t mb = xb_s + buf * W.kst2 * (NT * 128);   // this expert's mid tiles
        const uint32_t ms0 = tmem + XSFB_COL + buf * W.kst2 * 4;  // and their scale rows, in TMEM from here
        for (int kk = 0; kk < W.kst2; ++kk)
          tc_cp_sf(ms0 + kk * 4, sdesc_sf(xsf_s + (buf * W.kst2 + kk) * XSF_PITCH));
        for (int u = 0; u < U.n && ok; ++u) {
          if (!unit_has(U, u, i2, n_my2)) continue;
          const uint32_t d = acc_begin();
          if (d == 0xFFFFFFFFu) { ok = false; break; }
          for (int k0 = 0; k0 < W.kst2 && ok; k0 += KS2) {
            if (!(ok = wait_full())) break;
            const int nk = min(KS2, W.kst2 - k0);
            const uint32_t sb = smem_u32(stages + stage * STAGE_BYTES);
            const uint32_t sf0 = tmem + SF_COL0 + (it & 1) * SF_SLOT;
            for (int kk = 0; kk < nk; ++kk) tc_cp_sf(sf0 + kk * 8, sdesc_sf(sb + G2_SFA + kk * 512));
            for (int kk = 0; kk < nk; ++kk) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint32_t id = idesc_with_sf(IDESC2, ks, ks);
                mma_mxf8f6f4(d, sdesc_sw128(sb + kk * A_TILE + ks * 32),
                             sdesc_sw128(mb + (k0 + kk) * (NT * 128) + ks * 32), id, sf0 + kk * 8,
                             ms0 + (k0 + kk) * 4, (k0 > 0 || kk > 0 || ks > 0));
              }
            }
            release();
          }
          if (!ok) break;
          tc_commit(&S.accf[acc_n % NACC]);
          ++acc_n;
        }
        if (ok) tc_commit(&S.midempty[buf]);   // this expert's mid buffer may be refilled
      }
      if (!ok) { tc_commit(&S.accf[0]); const uint64_t until = globaltimer() + 2000000ull; while (globaltimer() < until) { } }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------ mid operand of GEMM2
    // Once every GEMM1 MMA has completed (their token operand's space is then
    // free), the warp polls the flags of all its (expert, k-block) mid tiles
    // with acquire loads, a lane per flag, keeping what it has seen; for each
    // of its experts in turn, once all k-blocks are published, lane 0 loads
    // the expert's 16 token rows of mid by TMA and their scale rows (stored
    // in the MMA's order by the publisher) by bulk copy into a free buffer.
    bool ok = mbar_wait(&S.g1done, 0, deadline, abort_flag);
    if (!ok && lane == 0) fail(4, 0);
    const int kst2 = W.kst2;
    const int nflags = n_my2 * kst2;   // flag f: expert slot f / kst2, k-block f % kst2
    uint32_t seen = 0;                 // bit q: flag lane + 32 q observed published
    auto poll = [&]() {                // acquire-load this lane's flags not seen yet
#pragma unroll 1
      for (int q = 0; q < 32; ++q) {
        const int f = lane + 32 * q;
        if (f >= nflags) break;
        if (!((seen >> q) & 1u) &&
            ld_acquire_gpu(p.flags + S.dlist[W.rank + (f / kst2) * CS] * MAX_J + f % kst2) == epoch)
          seen |= 1u << q;
      }
      __syncwarp();   // every lane's acquires before lane 0's loads of mid
    };
    auto expert_ready = [&](int i2) -> bool {   // warp-uniform
      bool r = true;
#pragma unroll 1
      for (int kk = 0; kk < kst2; ++kk) {
        const int f = i2 * kst2 + kk;
        r = r && ((__shfl_sync(0xFFFFFFFFu, seen, f & 31) >> (f >> 5)) & 1u);
      }
      return r;
    };
    for (int i2 = 0; i2 < n_my2 && ok; ++i2) {
      uint32_t spins = 0;
      while (!expert_ready(i2)) {
        poll();
        if ((++spins & 15u) == 0 && (*abort_flag || globaltimer() > deadline)) {
          if (lane == 0) fail(7, i2);
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (lane == 0) {
        const int e = S.dlist[W.rank + i2 * CS], buf = i2 % nbuf, use = i2 / nbuf;
        fence_proxy_async_global();   // the acquired mid is read by the async proxy
        if (!mbar_wait(&S.midempty[buf], (use & 1) ^ 1, deadline, abort_flag)) { fail(6, i2); ok = false; }
        if (ok) {
          mbar_arrive_expect_tx(&S.midfull[buf], kst2 * (NT * 128 + NT * 16));
          for (int kk = 0; kk < kst2; ++kk) {
            tma_load_2d(xb + (buf * kst2 + kk) * (NT * 128), &tmMid, &S.midfull[buf], kk * 128, e * NT);
            bulk_load(xsf + (buf * kst2 + kk) * XSF_PITCH, p.midsf + ((size_t)e * kst2 + kk) * 64, NT * 16,
                      &S.midfull[buf]);
          }
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    }
    if (!ok && lane == 0) { const uint64_t until = globaltimer() + 2000000ull; while (globaltimer() < until) { } }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue (warps 4..7)
    const int ew = warp - 4, row = 32 * ew + lane;   // TMEM lane quarter = warp % 4
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * ew) << 16);
    const uint32_t red_s = smem_u32(red);
    int acc_n = 0, red_n = 0;
    bool ok = true;
    // Barrier of the 128 epilogue threads.  Every wait of the kernel is
    // bounded, so a thread that gave up may skip an arrival; the others then
    // time out here instead of blocking in bar.sync for good.
    uint32_t epi_phase = 0;
    auto epi_bar = [&]() -> bool {
      mbar_arrive(&S.epibar);
      const bool got = mbar_wait(&S.epibar, epi_phase, deadline, abort_flag);
      epi_phase ^= 1;
      if (!got) fail(13, 0);
      return got;
    };
    // cross-rank reduction of `vals` (n floats per row) in rank order; rank 0
    // gets the sum.  Rank 0 issues all loads of a batch of peers before adding,
    // so a batch costs one distributed-shared-memory round trip.
    auto reduce = [&](float* vals, auto n_const) -> bool {
      constexpr int n = decltype(n_const)::value;
      constexpr int RB = (CS - 1) * (n / 4) <= 12 ? CS - 1 : 1;   // peers per batch (<= 12 float4 in flight)
      const int slot = red_n & 1;
      const uint32_t par = (red_n >> 1) & 1;
      ++red_n;
      if (W.rank != 0) {
        if (!mbar_wait_cluster(&S.red_free[slot], par ^ 1, deadline, abort_flag)) { fail(8, 0); return false; }
        float* dst = red + slot * RED_FLOATS + row * 32;
#pragma unroll
        for (int i = 0; i < n; i += 4)
          *reinterpret_cast<float4*>(dst + (((i >> 2) ^ (row & 7)) << 2)) =
              make_float4(vals[i], vals[i + 1], vals[i + 2], vals[i + 3]);
        if (!epi_bar()) return false;
        if (ew == 0 && lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.red_full[slot]), 0));
        return true;
      }
      if (!mbar_wait_cluster(&S.red_full[slot], par, deadline, abort_flag)) { fail(9, 0); return false; }
      const uint32_t mine = red_s + (slot * RED_FLOATS + row * 32) * 4;
#pragma unroll
      for (int r0 = 1; r0 < CS; r0 += RB) {
        float4 t[RB][n / 4];
#pragma unroll
        for (int rr = 0; rr < RB; ++rr) {
          const uint32_t src = mapa_shared(mine, r0 + rr);
#pragma unroll
          for (int i = 0; i < n / 4; ++i) t[rr][i] = ld_shared_cluster_f4(src + ((i ^ (row & 7)) << 4));
        }
#pragma unroll
        for (int rr = 0; rr < RB; ++rr)
#pragma unroll
          for (int i = 0; i < n / 4; ++i) {
            vals[4 * i] += t[rr][i].x; vals[4 * i + 1] += t[rr][i].y;
            vals[4 * i + 2] += t[rr][i].z; vals[4 * i + 3] += t[rr][i].w;
          }
      }
      if (!epi_bar()) return false;   // all rows read before the peers may overwrite
      if (ew == 0 && lane < CS && lane > 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.red_free[slot]), lane));
      return true;
    };
    for (int g = W.cid; g < W.ngroups && ok; g += W.ncl) {
      const int e = S.dlist[g / W.J], j = g % W.J;
      float v[2 * NTOK];   // gate of token t at v[t], up at v[NTOK + t], this row
      if (KR > 0) {
        const int b = acc_n % NACC;
        if (!mbar_wait(&S.accf[b], (acc_n / NACC) & 1, deadline, abort_flag)) { fail(10, 0); ok = false; break; }
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
        for (int i = 0; i < NTOK; ++i) { v[i] = gg[i]; v[NTOK + i] = uu[i]; }
      } else {
#pragma unroll
        for (int i = 0; i < 2 * NTOK; ++i) v[i] = 0.0f;
      }
      if (!reduce(v, std::integral_constant<int, 2 * NTOK>())) { ok = false; break; }
      if (W.rank != 0) continue;
      const int cnt = S.counts[e], off = S.offsets[e];
#pragma unroll
      for (int t = 0; t < NTOK; ++t)
        if (t < M) epi[t * 128 + row] = v[t] / (1.0f + expf(-v[t])) * v[NTOK + t];
      if (!epi_bar()) { ok = false; break; }
      for (int c = ew; c < cnt; c += 4) {   // mid quantized once per (pair, 128-block)
        const int t = S.sorted_tok[off + c];
        const float4 q4 = reinterpret_cast<const float4*>(epi + t * 128)[lane];
        float amax = fmaxf(fmaxf(fabsf(q4.x), fabsf(q4.y)), fmaxf(fabsf(q4.z), fabsf(q4.w)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const int ke = pow2_e4m3_exp(amax);
        const float inv = exp2i(-ke);
        const size_t r = (size_t)(off + c);
        const uint32_t q = cvt_e4m3x4(q4.x * inv, q4.y * inv, q4.z * inv, q4.w * inv);
        reinterpret_cast<uint32_t*>(p.midq + r * I + j * 128)[lane] = q;                    // sorted-pair tap
        reinterpret_cast<uint32_t*>(p.midt + ((size_t)e * NT + t) * I + j * 128)[lane] = q; // GEMM2 operand row t
        if (lane == 0) {
          p.midqs[r * (I / 128) + j] = exp2i(ke);
          p.midsf[((size_t)e * W.J + j) * 64 + t * 4] = rep4((uint32_t)(ke + 127));   // B scale row t, E8M0
        }
      }
      if (!epi_bar()) { ok = false; break; }   // the 4 warps' stores before the release (gpu scope, cumulative)
      // (the test knob withholds the call's first flag, so that the waits on it run out)
      if (ew == 0 && lane == 0 && !(p.test_withhold && g == 0)) st_release_gpu(p.flags + e * MAX_J + j, epoch);
    }
    float acc[2][NTOK];   // unit n of this cluster, token t (items run expert-major)
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int i = 0; i < NTOK; ++i) acc[n][i] = 0.0f;
    for (int i2 = 0; i2 < n_my2 && ok; ++i2) {
      const float4* wt = reinterpret_cast<const float4*>(S.wtok[i2]);
      for (int n = 0; n < U.n && ok; ++n) {
        if (!unit_has(U, n, i2, n_my2)) continue;
        const int b = acc_n % NACC;
        if (!mbar_wait(&S.accf[b], (acc_n / NACC) & 1, deadline, abort_flag)) { fail(10, 1); ok = false; break; }
        tc_fence_after();
        float y[16];   // column t: token t's row of mid times this w2 tile
        tmem_ld16(tl + b * 32, y);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acce[b]);
        ++acc_n;
#pragma unroll
        for (int nn = 0; nn < 2; ++nn) {
          if (nn != n) continue;
#pragma unroll
          for (int q = 0; q < NTOK / 4; ++q) {   // columns of tokens that did not pick this expert are skipped
            const float4 w = wt[q];
            if (w.x != 0.0f) acc[nn][4 * q] = fmaf(w.x, y[4 * q], acc[nn][4 * q]);
            if (w.y != 0.0f) acc[nn][4 * q + 1] = fmaf(w.y, y[4 * q + 1], acc[nn][4 * q + 1]);
            if (w.z != 0.0f) acc[nn][4 * q + 2] = fmaf(w.z, y[4 * q + 2], acc[nn][4 * q + 2]);
            if (w.w != 0.0f) acc[nn][4 * q + 3] = fmaf(w.w, y[4 * q + 3], acc[nn][4 * q + 3]);
          }
        }
      }
    }
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      if (n >= U.n || !ok) break;
      if (!reduce(acc[n], std::integral_constant<int, NTOK>())) { ok = false; break; }
      if (W.rank != 0) continue;
      const int ht = U.ht[n], half = U.half[n];
      float* xp = p.xpart + ((size_t)ht * 128 + row) * NT;   // this row's partial of a split h-tile
      if (half == 2) {   // partner: hand the half's sum to the owner
#pragma unroll
        for (int t = 0; t < NTOK; t += 4)
          __stcg(reinterpret_cast<float4*>(xp + t), make_float4(acc[n][t], acc[n][t + 1], acc[n][t + 2], acc[n][t + 3]));
        if (!epi_bar()) { ok = false; break; }   // every row stored before the release (gpu scope, cumulative)
        if (ew == 0 && lane == 0) st_release_gpu(p.xflag + ht, epoch);
        continue;
      }
      if (half == 1) {   // owner: add the partner's half after its own
        if (ew == 0 && lane == 0) {
          int got = 1;
          uint32_t spins = 0;
          while (ld_acquire_gpu(p.xflag + ht) != epoch)
            if ((++spins & 63u) == 0 && (*abort_flag || globaltimer() > deadline)) { fail(12, ht); got = 0; break; }
          S.xok = got;
        }
        if (!epi_bar() || !S.xok) { ok = false; break; }
#pragma unroll
        for (int t = 0; t < NTOK; t += 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(xp + t));
          acc[n][t] += v.x; acc[n][t + 1] += v.y; acc[n][t + 2] += v.z; acc[n][t + 3] += v.w;
        }
      }
      for (int t = 0; t < M; ++t) {
        if (p.out_f32) {
          p.out_f32[(size_t)t * H + ht * 128 + row] = acc[n][t];
        } else {
          const uint32_t b2 = pack_bf16x2(acc[n][t], 0.0f) & 0xFFFFu;
          p.out[(size_t)t * H + ht * 128 + row] = static_cast<uint16_t>(b2);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == NWARPS - 1) {   // the allocating warp releases the columns
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
template <int NTOK>
static void small_set_smem() {
  cudaFuncSetAttribute(k_moe_small<NTOK>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
}

static void small_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, int nclusters, cudaStream_t st) {
  *cfg = cudaLaunchConfig_t{};
  cfg->gridDim = dim3(nclusters * CS);
  cfg->blockDim = dim3(THREADS);
  cfg->dynamicSmemBytes = SMEM_BYTES;
  cfg->stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}

int small_cluster_size() { return CS; }

int small_max_clusters(int dev) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    small_set_smem<4>(); small_set_smem<8>(); small_set_smem<12>(); small_set_smem<16>();
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    small_config(&cfg, attr, 1, 0);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_moe_small<16>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = -1;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

cudaError_t launch_small(const CUtensorMap& w13, const CUtensorMap& w2, const CUtensorMap& mid,
                         const SmallParams& p, int nclusters, cudaStream_t st) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  small_config(&cfg, attr, nclusters, st);
  if (p.M <= 4) return cudaLaunchKernelEx(&cfg, k_moe_small<4>, w13, w2, mid, p);
  if (p.M <= 8) return cudaLaunchKernelEx(&cfg, k_moe_small<8>, w13, w2, mid, p);
  if (p.M <= 12) return cudaLaunchKernelEx(&cfg, k_moe_small<12>, w13, w2, mid, p);
  return cudaLaunchKernelEx(&cfg, k_moe_small<16>, w13, w2, mid, p);
}

}  // namespace moe
