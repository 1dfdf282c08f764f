// gemm.cu -- the two grouped, block-scaled expert GEMMs on the 5th-generation
// tensor cores (tcgen05), expert-major.
//
// GEMM1 (up/gate) + SwiGLU + mid quantization, and GEMM2 (down), are one
// persistent, warp-specialized kernel template.  Weights are the MMA's M side
// (128 weight rows per instruction), the pairs routed to one expert its N side
// (16..64 rows): every expert's weight tile is streamed from HBM once for all
// the pairs that picked it ("glm53_flash: score a verify request's index tiles
// once", commit message: expert-major above 8 rows).
//
//   warp 0      producer: weight tiles (TMA, 3-D tensor map [E][rows][K]), a
//               2-D tile of the token rows (GEMM1: copied into sorted-pair
//               order after the sort) or of mid (GEMM2), and the stage's
//               scale-factor blocks by bulk copy, all
//               stored ahead of time in the order the tensor cores read them
//               (weights: moe_pack_mxfp4_scales; tokens: packed per token
//               tile after the sort; mid: packed by GEMM1's epilogue)
//   warp 1      TMEM owner; lane 0 issues tcgen05.cp (scale factors) + tcgen05.mma
//   warps 2..   epilogue: TMEM -> registers; GEMM1: SwiGLU, per-(pair, 128)
//               power-of-two E4M3 quantization of mid, written once ("glm53:
//               FP8 mid hand-off", Modifications table row 1); GEMM2: each
//               pair's row y times its routing weight, rounded once to bf16
//               (the combine adds the k rows of a token).
//
// Formats:
//   MXFP4 GEMM1  kind::mxf4      A = w13 E2M1, B = x E2M1, E8M0 per 32 on both
//   MXFP4 GEMM2  kind::mxf8f6f4  A = w2 E2M1 (TMA-unpacked to a byte each),
//                                B = mid E4M3, its power-of-two scale as E8M0
//   FP8 GEMM1/2  kind::mxf8f6f4  E4M3 x E4M3; the activation/mid power-of-two
//                scale rides in the MMA (B scale factor), the fp32 128x128 weight
//                block scale is applied per 128-K block by the epilogue
//                ("promotion"): each K block lands in its own TMEM partial.
//
// Block-FP8 calls with 32 or more pairs per expert use the wide variant at the
// end of this file (k_gemm_wide): pairs on M, 256 weight rows on N.
//
// Every mbarrier wait is bounded; on timeout the CTA records ST_TIMEOUT in the
// status word and unwinds.
#include "codec.cuh"

namespace moe {

enum GemmKind : int { G1_MX = 0, G1_F8 = 1, G2_MX = 2, G2_F8 = 3 };

template <int KIND, int NT, int STAGES>
struct GCfg {
  static constexpr bool G1 = (KIND == G1_MX || KIND == G1_F8);
  static constexpr bool F8 = (KIND == G1_F8 || KIND == G2_F8);
  // A tiles per stage: GEMM1 a gate and an up tile of w13, GEMM2 two
  // consecutive 128-row h-tiles of w2 (a task covers 256 rows of the output)
  static constexpr int NA = 2;
  static constexpr int CH = (KIND == G1_MX) ? 2 : 1;     // 128-element scale chunks per stage
  static constexpr int A_BYTES = kTileW * kStageBytesK;  // 16 KB
  static constexpr int B_BYTES = NT * kStageBytesK;
  static constexpr int SF_CHUNK = 512;
  static constexpr int OFF_B = NA * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + NA * CH * SF_CHUNK;
  static constexpr int STAGE_BYTES = (OFF_SFB + CH * SF_CHUNK + 1023) & ~1023;
  static constexpr int EPI_WARPS = F8 ? 8 : 4;
  // promotion path: two warps share a 32-lane quarter and split the columns
  // (16-column loads), except at NT = 16 where the second warp only keeps
  // the barrier counts
  static constexpr int HALVES = (F8 && NT >= 32) ? 2 : 1;
  static constexpr int CPW = NT / HALVES;
  static constexpr int EPI_THREADS = EPI_WARPS * 32;
  static constexpr int THREADS = 64 + EPI_THREADS;       // producer, MMA, epilogue warps
  // GEMM1: the SwiGLU tile (fp32); GEMM2: one bf16 staging tile per epilogue
  // warp and h-tile (32 rows x its columns), so the output leaves in 16-byte stores
  static constexpr int EPI_BYTES = G1 ? NT * 128 * 4 : EPI_WARPS * NA * 32 * CPW * 2;
  static constexpr int ACC_COLS = NA * NT;               // TMEM columns of one accumulator set
  // block-FP8: per-128-K partials, up to 4 in flight so the MMA runs ahead of
  // the promotion; otherwise two whole-task accumulators
  static constexpr int SF_COL0 = F8 ? 384 : 256;
  static constexpr int NPART = F8 ? (SF_COL0 / ACC_COLS < 4 ? SF_COL0 / ACC_COLS : 4) : 2;
  static constexpr int SF_SLOT_COLS = (NA + 1) * CH * 4;
  // block-FP8: the weights' scale factors (all 2^0) live in TMEM for the whole kernel
  static constexpr int SF_FIX = SF_COL0 + 2 * SF_SLOT_COLS;
  // bytes the copy engine reports per stage: the unpacked 4-bit operand counts
  // its packed global bytes (half of its shared-memory footprint); MXFP4
  // weight scale blocks and the operand's scale blocks arrive by bulk copy
  // (block-FP8 weight scales are applied by the epilogue instead)
  static constexpr uint32_t TX = NA * (KIND == G2_MX ? A_BYTES / 2 : A_BYTES) + B_BYTES +
                                 (F8 ? 0 : NA * CH * SF_CHUNK) + CH * SF_CHUNK;
  static constexpr uint32_t IDESC =
      KIND == G1_MX ? idesc_block_scaled(FMT4_E2M1, FMT4_E2M1, NT)
    : KIND == G2_MX ? idesc_block_scaled(FMT8_E2M1, FMT8_E4M3, NT)
                    : idesc_block_scaled(FMT8_E4M3, FMT8_E4M3, NT);
  static constexpr int TABLE_INTS = kMaxE + 8;           // one per-expert table
  static constexpr int SMEM = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 3 * TABLE_INTS * 4 + 1024;
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 64, "token tile");
  static_assert(NPART >= 2 && NPART * ACC_COLS <= SF_COL0, "accumulators overlap scale factors");
  static_assert(SF_FIX + NA * CH * 4 <= 512, "TMEM columns");
  static_assert(SMEM <= 232448, "shared memory");
};

struct Task {
  int e, tt, j, s, row0, valid, k0, k1, group, tile;
};

// Per-expert tables of the call, staged in shared memory at kernel start so
// that decoding a task costs a few shared-memory reads, not a chain of
// dependent global loads.
struct Tables {
  const int* tiles;    // [E+1] prefix of token tiles per expert
  const int* offsets;  // [E+1] first sorted pair of each expert
  const int* counts;   // [E]   pairs per expert
};

// Task order: expert-major; inside an expert, (n-tile, split) blocks, and the
// token tiles of one weight tile adjacent so they run concurrently (L2 reuse).
__device__ __forceinline__ void decode_task(const GemmParams& p, const Tables& tb_s, int idx, int nt, bool g1,
                                            Task& t) {
  const int mult = g1 ? p.jn * p.split : p.jn;
  int lo = 0, hi = p.E;  // largest e with tiles[e] * mult <= idx
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tb_s.tiles[mid] * mult <= idx) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int tb = tb_s.tiles[e];
  const int ntiles = tb_s.tiles[e + 1] - tb;
  const int local = idx - tb * mult;
  t.e = e;
  t.tt = local % ntiles;
  const int js = local / ntiles;
  if (g1) { t.s = js % p.split; t.j = js / p.split; } else { t.s = 0; t.j = js; }
  t.row0 = tb_s.offsets[e] + t.tt * nt;
  t.valid = min(nt, tb_s.counts[e] - t.tt * nt);
  const int per = p.kst / p.split;
  t.k0 = t.s * per;
  t.k1 = t.k0 + per;
  t.group = (tb + t.tt) * p.jn + t.j;
  t.tile = tb + t.tt;
}

// silu(g) * u with the fast exponential and an approximate reciprocal (the
// result feeds a quantization to E4M3, whose step is far coarser than their
// error; for g below about -88 the denominator is +inf and the result 0)
__device__ __forceinline__ float silu_mul(float g, float u) { return g * rcp_approx(1.0f + __expf(-g)) * u; }

// Wait sites, recorded with the first timeout of a call.
enum : int { W_PROD_EMPTY = 1, W_MMA_ACCE = 2, W_MMA_FULL = 3, W_MMA_PEMPTY = 4, W_EPI_ACCF = 6 };

__device__ __forceinline__ void flag_timeout(const GemmParams& p, volatile int* abort_flag, int kind, int site,
                                             int kst) {
  *abort_flag = 1;
  atomicOr(p.status, ST_TIMEOUT);
  const int code = (int)(0x80000000u | ((unsigned)kind << 24) | ((unsigned)site << 20) |
                         ((unsigned)min(kst, 255) << 12) | (blockIdx.x & 0xFFFu));
  atomicCAS(p.status + 2, 0, code);
}

template <int KIND, int NT, int STAGES>
__global__ void __launch_bounds__(GCfg<KIND, NT, STAGES>::THREADS, 1)
k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
       const GemmParams p) {
  using C = GCfg<KIND, NT, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  float* epi = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES + C::EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;     // accumulator (or K-block partial) full
  uint64_t* acce = accf + 4;           // ... and drained by the epilogue
  uint64_t* epibar = acce + 4;         // the epilogue threads' barrier (bounded, unlike bar.sync)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(epibar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* sh_last = abort_flag + 1;
  int* tab = reinterpret_cast<int*>(smem + STAGES * C::STAGE_BYTES + C::EPI_BYTES + 1024);
  const Tables tbl{tab, tab + C::TABLE_INTS, tab + 2 * C::TABLE_INTS};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < C::NPART; ++b) { mbar_init(&accf[b], 1); mbar_init(&acce[b], C::EPI_WARPS); }
    mbar_init(epibar, C::EPI_THREADS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB); }
  if (warp == 1) { tmem_alloc(tmem_holder, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_wait();  // inputs of this step are complete and visible
  pdl_launch_dependents();
  for (int i = threadIdx.x; i <= p.E; i += C::THREADS) {
    tab[i] = __ldcg(p.tiles + i);
    tab[C::TABLE_INTS + i] = __ldcg(p.offsets + i);
    tab[2 * C::TABLE_INTS + i] = i < p.E ? __ldcg(p.counts + i) : 0;
  }
  if (C::F8 && warp >= 2) {
    // block-FP8 weights: the MMA's weight scale factors are all 2^0 (the
    // epilogue applies the fp32 block scales), written once into every stage
    constexpr int WORDS = C::NA * C::CH * C::SF_CHUNK / 4;
    for (int i = threadIdx.x - 64; i < STAGES * WORDS; i += C::EPI_THREADS)
      reinterpret_cast<uint32_t*>(stages + (i / WORDS) * C::STAGE_BYTES + C::OFF_SFA)[i % WORDS] = 0x7F7F7F7Fu;
    fence_proxy_async_smem();
  }
  __syncthreads();

  const int mult = C::G1 ? p.jn * p.split : p.jn;
  const int total = tbl.tiles[p.E] * mult;
  const uint64_t deadline = globaltimer() + p.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    for (int idx = blockIdx.x; idx < total; idx += gridDim.x) {
      Task t;
      decode_task(p, tbl, idx, NT, C::G1, t);
      bool ok = true;
      int kfail = 0;
      for (int kst = t.k0; kst < t.k1; ++kst) {
        if (!mbar_wait(&empty[stage], phase ^ 1, deadline, abort_flag)) { ok = false; kfail = kst; break; }
        if (lane == 0) {
          uint8_t* sb = stages + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::TX);
          if (C::G1) {
            tma_load_3d(sb, &tmA, &full[stage], kst * kStageBytesK, t.j * kTileW, t.e);
            tma_load_3d(sb + C::A_BYTES, &tmA, &full[stage], kst * kStageBytesK, p.I + t.j * kTileW, t.e);
            tma_load_2d(sb + C::OFF_B, &tmB, &full[stage], kst * kStageBytesK, t.row0);
          } else {
            // GEMM2: K coordinate in elements (128 per stage) for both formats; the
            // second h-tile of an odd count lies past H (zero-filled, not stored)
            tma_load_3d(sb, &tmA, &full[stage], kst * 128, 2 * t.j * kTileW, t.e);
            tma_load_3d(sb + C::A_BYTES, &tmA, &full[stage], kst * 128, (2 * t.j + 1) * kTileW, t.e);
            tma_load_2d(sb + C::OFF_B, &tmB, &full[stage], kst * 128, t.row0);
          }
          if (!C::F8) {
            // packed MXFP4 weight scales: the stage's 128-column blocks of each tile are contiguous
            if (C::G1) {
              const size_t rt = p.H / 128;   // blocks per 128-row tile of w13
              bulk_load(sb + C::OFF_SFA, p.sfa_u8 + (((size_t)t.e * (2 * p.I / 128) + t.j) * rt + kst * 2) * 512,
                        2 * C::SF_CHUNK, &full[stage]);
              bulk_load(sb + C::OFF_SFA + 2 * C::SF_CHUNK,
                        p.sfa_u8 + (((size_t)t.e * (2 * p.I / 128) + p.I / 128 + t.j) * rt + kst * 2) * 512,
                        2 * C::SF_CHUNK, &full[stage]);
            } else {
              const int ht = p.H / 128;
#pragma unroll
              for (int a = 0; a < 2; ++a)
                bulk_load(sb + C::OFF_SFA + a * C::SF_CHUNK,
                          p.sfa_u8 + (((size_t)t.e * ht + min(2 * t.j + a, ht - 1)) * (p.I / 128) + kst) * 512,
                          C::SF_CHUNK, &full[stage]);
            }
          }
          // the token tile's operand scales, packed per (tile, 128-column chunk)
          bulk_load(sb + C::OFF_SFB, p.bsf + ((size_t)t.tile * p.nchb + kst * C::CH) * 512, C::CH * C::SF_CHUNK,
                    &full[stage]);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      __syncwarp();
      if (!ok) {
        if (lane == 0) flag_timeout(p, abort_flag, KIND, W_PROD_EMPTY, kfail);
        // let copies already issued land before the CTA's shared memory goes away
        const uint64_t until = globaltimer() + 2000000ull;
        while (globaltimer() < until) { }
        break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, it = 0, tcount = 0, kb_it = 0, site = 0, kfail = 0;
      if (C::F8)   // the constant weight scale factors, once (every stage holds the same 2^0 blocks)
        for (int i = 0; i < C::NA * C::CH; ++i)
          tc_cp_sf(tmem + C::SF_FIX + i * 4, sdesc_sf(smem_u32(stages + C::OFF_SFA + i * 512)));
      uint32_t phase = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        Task t;
        decode_task(p, tbl, idx, NT, C::G1, t);
        const int b = tcount & 1;
        if (!C::F8) {
          if (!mbar_wait(&acce[b], ((tcount >> 1) & 1) ^ 1, deadline, abort_flag)) {
            ok = false; site = W_MMA_ACCE; kfail = t.k0; break;
          }
          tc_fence_after();
        }
        for (int kst = t.k0; kst < t.k1; ++kst) {
          if (!mbar_wait(&full[stage], phase, deadline, abort_flag)) { ok = false; site = W_MMA_FULL; kfail = kst; break; }
          tc_fence_after();
          uint8_t* sb = stages + stage * C::STAGE_BYTES;
          const uint32_t sf0 = tmem + C::SF_COL0 + (it & 1) * C::SF_SLOT_COLS;
          if (!C::F8) {
#pragma unroll
            for (int a = 0; a < C::NA; ++a)
#pragma unroll
              for (int c = 0; c < C::CH; ++c)
                tc_cp_sf(sf0 + (a * C::CH + c) * 4, sdesc_sf(smem_u32(sb + C::OFF_SFA + (a * C::CH + c) * 512)));
          }
#pragma unroll
          for (int c = 0; c < C::CH; ++c)
            tc_cp_sf(sf0 + (C::NA * C::CH + c) * 4, sdesc_sf(smem_u32(sb + C::OFF_SFB + c * 512)));
          uint32_t d0;
          int pb = 0;
          if (C::F8) {
            pb = kb_it % C::NPART;
            if (!mbar_wait(&acce[pb], ((kb_it / C::NPART) & 1) ^ 1, deadline, abort_flag)) {
              ok = false; site = W_MMA_PEMPTY; kfail = kst; break;
            }
            tc_fence_after();
            d0 = tmem + pb * C::ACC_COLS;
          } else {
            d0 = tmem + b * C::ACC_COLS;
          }
          const uint32_t a_base = smem_u32(sb), b_base = smem_u32(sb + C::OFF_B);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const int c = (KIND == G1_MX) ? (ks >> 1) : 0;
            const uint32_t sfid = (KIND == G1_MX) ? (ks & 1) * 2 : ks;
            const uint32_t idesc = idesc_with_sf(C::IDESC, sfid, sfid);
            const uint32_t acc = C::F8 ? (ks > 0) : (kst > t.k0 || ks > 0);
            const uint64_t bdesc = sdesc_sw128(b_base + ks * 32);
#pragma unroll
            for (int a = 0; a < C::NA; ++a) {
              const uint64_t adesc = sdesc_sw128(a_base + a * C::A_BYTES + ks * 32);
              const uint32_t sfa = (C::F8 ? tmem + C::SF_FIX : sf0) + (a * C::CH + c) * 4;
              const uint32_t sfb = sf0 + (C::NA * C::CH + c) * 4;
              if (KIND == G1_MX) mma_mxf4(d0 + a * NT, adesc, bdesc, idesc, sfa, sfb, acc);
              else mma_mxf8f6f4(d0 + a * NT, adesc, bdesc, idesc, sfa, sfb, acc);
            }
          }
          tc_commit(&empty[stage]);
          if (C::F8) { tc_commit(&accf[pb]); ++kb_it; }
          ++it;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (!C::F8) tc_commit(&accf[b]);
        ++tcount;
      }
      if (!ok) {
        flag_timeout(p, abort_flag, KIND, site, kfail);
        // drain this thread's tensor-core work before TMEM is released
        tc_commit(&accf[0]);
        const uint64_t until = globaltimer() + 2000000ull;
        while (globaltimer() < until) { }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue
    const int ew = warp - 2, q = warp & 3, half = ew >> 2;   // q: the warp's TMEM lane quarter
    const int row = 32 * q + lane;                     // weight row inside the tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16);
    int tcount = 0, kb_it = 0, kfail = 0;
    bool ok = true;
    // Every wait of the kernel is bounded, so a thread that gave up may miss
    // an arrival here; the others then time out instead of blocking in bar.sync.
    uint32_t epi_phase = 0;
    auto epi_bar = [&]() -> bool {
      mbar_arrive(epibar);
      const bool got = mbar_wait(epibar, epi_phase, deadline, abort_flag);
      epi_phase ^= 1;
      return got;
    };
    // block-FP8 weight scales of a task (one per 128-K block and A tile),
    // kept in registers spread over the lanes when the task has <= 64 K blocks
    constexpr int SWR = 2;
    float swc[C::NA][SWR], swn[C::NA][SWR];
    const bool sw_in_regs = (p.kst / p.split) <= 32 * SWR;
    auto sw_ptr = [&](const Task& tt, int a, int kb) -> const float* {
      if (C::G1)
        return p.sfa_f32 + ((size_t)tt.e * (2 * p.I / 128) + (a ? p.I / 128 : 0) + tt.j) * (p.H / 128) + kb;
      return p.sfa_f32 + ((size_t)tt.e * (p.H / 128) + min(2 * tt.j + a, p.H / 128 - 1)) * (p.I / 128) + kb;
    };
    auto load_sw = [&](int idx, float (&dst)[C::NA][SWR]) {
      if (!C::F8 || !sw_in_regs || idx >= total) return;
      Task tn;
      decode_task(p, tbl, idx, NT, C::G1, tn);
#pragma unroll
      for (int a = 0; a < C::NA; ++a)
#pragma unroll
        for (int r = 0; r < SWR; ++r) {
          const int kb = tn.k0 + lane + 32 * r;
          dst[a][r] = kb < tn.k1 ? __ldg(sw_ptr(tn, a, kb)) : 0.0f;
        }
    };
#pragma unroll
    for (int a = 0; a < C::NA; ++a)
#pragma unroll
      for (int r = 0; r < SWR; ++r) { swc[a][r] = 0.0f; swn[a][r] = 0.0f; }
    load_sw(blockIdx.x, swn);
    // GEMM2: routing weight of each token column (column c in lane c % 32,
    // register c / 32), loaded a task ahead; GEMM2 writes bf16(w * y)
    float wc[2] = {0.0f, 0.0f}, wn[2] = {0.0f, 0.0f};
    auto load_w = [&](int idx, float (&dst)[2]) {
      if (C::G1 || idx >= total) return;
      Task tn;
      decode_task(p, tbl, idx, NT, C::G1, tn);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int c = lane + 32 * r;
        dst[r] = c < tn.valid ? __ldcg(p.sorted_w + tn.row0 + c) : 0.0f;
      }
    };
    load_w(blockIdx.x, wn);
    // GEMM2: this warp's 32 rows x CPW columns of bf16(w * y), column-major in
    // shared memory, leave as 16-byte stores (4 lanes per 64-byte column
    // segment); columns past the expert's last pair are not written
    uint16_t* stg = reinterpret_cast<uint16_t*>(epi) + ew * C::NA * 32 * C::CPW;   // [h-tile][column][32 rows]
    auto store_tile = [&](const Task& tt, int col0) {
      __syncwarp();
#pragma unroll
      for (int a = 0; a < C::NA; ++a) {
        const int ht = 2 * tt.j + a;
        if (ht * kTileW >= p.H) break;
#pragma unroll
        for (int i = 0; i < C::CPW / 8; ++i) {
          const int k = lane + 32 * i, cl = k >> 2, part = k & 3, c = col0 + cl;
          const uint4 v = *reinterpret_cast<const uint4*>(stg + (a * C::CPW + cl) * 32 + part * 8);
          if (c < tt.valid)
            *reinterpret_cast<uint4*>(p.yw + (size_t)(tt.row0 + c) * p.H + ht * kTileW + 32 * q + part * 8) = v;
        }
      }
      __syncwarp();
    };
    for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x, ++tcount) {
      Task t;
      decode_task(p, tbl, idx, NT, C::G1, t);
      if (!C::G1) {
        wc[0] = wn[0]; wc[1] = wn[1];
        load_w(idx + (int)gridDim.x, wn);
      }
      const int b = tcount & 1;
      if (!C::F8) {
        if (!mbar_wait(&accf[b], (tcount >> 1) & 1, deadline, abort_flag)) { ok = false; kfail = t.k0; break; }
        tc_fence_after();
        const uint32_t base = tl + b * C::ACC_COLS;
#pragma unroll
        for (int cc = 0; cc < NT / 16; ++cc) {
          float g[16], u[16];   // GEMM1: gate, up; GEMM2: the two h-tiles
          tmem_ld16(base + cc * 16, g);
          tmem_ld16(base + NT + cc * 16, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = cc * 16 + i;
            if (C::G1) {
              if (p.split == 1) {
                epi[c * 128 + row] = silu_mul(g[i], u[i]);
              } else {
                float* dst = p.part + ((size_t)(t.group * p.split + t.s) * NT + c) * 256;
                dst[row] = g[i];
                dst[128 + row] = u[i];
              }
            } else {
              const float w = __shfl_sync(0xFFFFFFFFu, c < 32 ? wc[0] : wc[1], c & 31);
              stg[c * 32 + lane] = bf16_bits(w * g[i]);
              stg[(C::CPW + c) * 32 + lane] = bf16_bits(w * u[i]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[b]);
        if (!C::G1) store_tile(t, 0);
      } else {
        // promotion: acc += s_w(K block) * partial(K block).  The weight
        // block scales of the task were loaded a task ahead, spread over the
        // warp's lanes (K block q of the task in lane q % 32, register q / 32).
        float acc[C::NA][C::CPW];
#pragma unroll
        for (int a = 0; a < C::NA; ++a)
#pragma unroll
          for (int i = 0; i < C::CPW; ++i) acc[a][i] = 0.0f;
#pragma unroll
        for (int a = 0; a < C::NA; ++a)
#pragma unroll
          for (int r = 0; r < SWR; ++r) swc[a][r] = swn[a][r];
        load_sw(idx + (int)gridDim.x, swn);
        const bool cols = half < C::HALVES;
        for (int kst = t.k0; kst < t.k1; ++kst, ++kb_it) {
          const int pb = kb_it % C::NPART;
          float sw[C::NA];
#pragma unroll
          for (int a = 0; a < C::NA; ++a) {
            const int q = kst - t.k0;
            sw[a] = sw_in_regs ? __shfl_sync(0xFFFFFFFFu, (q >> 5) ? swc[a][1] : swc[a][0], q & 31)
                               : __ldg(sw_ptr(t, a, kst));
          }
          if (!mbar_wait(&accf[pb], (kb_it / C::NPART) & 1, deadline, abort_flag)) { ok = false; kfail = kst; break; }
          tc_fence_after();
          if (cols) {
#pragma unroll
            for (int a = 0; a < C::NA; ++a) {
              float v[C::CPW];
              if constexpr (C::CPW == 32) {
                tmem_ld32(tl + pb * C::ACC_COLS + a * NT + half * C::CPW, v);
              } else {
#pragma unroll
                for (int cc = 0; cc < C::CPW / 16; ++cc)
                  tmem_ld16(tl + pb * C::ACC_COLS + a * NT + half * C::CPW + cc * 16,
                            *reinterpret_cast<float(*)[16]>(v + cc * 16));
              }
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < C::CPW; ++i) acc[a][i] = fmaf(sw[a], v[i], acc[a][i]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acce[pb]);
        }
        if (!ok) break;
        if (cols) {
#pragma unroll
          for (int i = 0; i < C::CPW; ++i) {
            const int c = half * C::CPW + i;
            if (C::G1) {
              epi[c * 128 + row] = silu_mul(acc[0][i], acc[C::NA - 1][i]);
            } else {
              const float w = __shfl_sync(0xFFFFFFFFu, c < 32 ? wc[0] : wc[1], c & 31);
              stg[i * 32 + lane] = bf16_bits(w * acc[0][i]);
              stg[(C::CPW + i) * 32 + lane] = bf16_bits(w * acc[1][i]);
            }
          }
          if (!C::G1) store_tile(t, half * C::CPW);
        }
      }
      if (C::G1) {
        if (!C::F8 && p.split > 1) {
          // split-K: the last of the splits to arrive sums them in split order
          __threadfence();
          if (!epi_bar()) { ok = false; break; }
          if (ew == 0 && lane == 0) {
            const int old = atomicAdd(p.cnt + t.group, 1);
            const int last = (old == p.split - 1);
            if (last) atomicExch(p.cnt + t.group, 0);
            *sh_last = last;
          }
          if (!epi_bar()) { ok = false; break; }
          if (!*sh_last) continue;
          __threadfence();
          // float4 of 4 weight rows per item, all splits' loads in flight at once
          const int et = threadIdx.x - 64;
#pragma unroll
          for (int it2 = 0; it2 < NT * 32 / C::EPI_THREADS; ++it2) {
            const int item = et + it2 * C::EPI_THREADS;
            const int c = item >> 5, r4 = (item & 31) * 4;
            float4 g4[8], u4[8];
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
              if (s2 < p.split) {
                const float* src = p.part + ((size_t)(t.group * p.split + s2) * NT + c) * 256;
                g4[s2] = __ldcg(reinterpret_cast<const float4*>(src + r4));
                u4[s2] = __ldcg(reinterpret_cast<const float4*>(src + 128 + r4));
              }
            }
            float4 g = g4[0], u = u4[0];
#pragma unroll
            for (int s2 = 1; s2 < 8; ++s2) {
              if (s2 < p.split) {
                g.x += g4[s2].x; g.y += g4[s2].y; g.z += g4[s2].z; g.w += g4[s2].w;
                u.x += u4[s2].x; u.y += u4[s2].y; u.z += u4[s2].z; u.w += u4[s2].w;
              }
            }
            float* dst = epi + c * 128 + r4;
            dst[0] = silu_mul(g.x, u.x); dst[1] = silu_mul(g.y, u.y);
            dst[2] = silu_mul(g.z, u.z); dst[3] = silu_mul(g.w, u.w);
          }
        }
        if (!epi_bar()) { ok = false; break; }
        // mid quantized once per (pair, 128-block): power-of-two scale, E4M3
        for (int c = ew; c < t.valid; c += C::EPI_WARPS) {
          const float4 v = reinterpret_cast<const float4*>(epi + c * 128)[lane];
          float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
          const int ke = pow2_e4m3_exp(amax);
          const float inv = exp2i(-ke);
          const uint32_t qv = cvt_e4m3x4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
          const size_t r = (size_t)(t.row0 + c);
          reinterpret_cast<uint32_t*>(p.midq + r * p.I + t.j * kTileW)[lane] = qv;
          if (lane == 0) {
            p.midqs[r * (p.I / 128) + t.j] = exp2i(ke);
            // GEMM2's operand scale for this pair and 128-block, packed like the token scales
            p.bsf_out[((size_t)t.tile * (p.I / 128) + t.j) * 128 + 4 * (c % 32) + c / 32] = rep4((uint32_t)(ke + 127));
          }
        }
        if (!epi_bar()) { ok = false; break; }
      }
    }
    if (!ok && lane == 0) flag_timeout(p, abort_flag, KIND, W_EPI_ACCF, kfail);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Block-FP8, wide tiles: once the experts hold 32 or more pairs on average,
// 128 sorted pairs are the MMA's M side and 256 weight rows its N side
// (GEMM1: a gate and an up tile of one 128-row n-tile; GEMM2: two h-tiles).
// A stage then carries 16 KB of pairs and 32 KB of weights for a 128 x 256 x
// 128 block, 24 KB per 128^3 against 40 KB in the weights-on-M layout, so
// the same four-stage ring in shared memory feeds twice the tensor work.
//
// The MMA takes plain E4M3 x E4M3 (kind::f8f6f4).  Both scales of a K block
// are per-thread scalars of the promotion: the weights' fp32 128x128 block
// scale is one per A-tile (column half) and the operand's power-of-two scale
// one per pair, i.e. per TMEM lane; their product is exact.  Each K block
// lands in one of two 256-column TMEM partials.  The epilogue warps own 32
// pairs (their TMEM lane quarter) times 64 columns of each half.  The pairs'
// scale blocks reach the epilogue through their own ring in shared memory
// (one 512-byte block per K block, filled by the producer's bulk copies), so
// no global load sits in the promotion loop.
template <bool G1>
struct WCfg {
  static constexpr int BM = 128;                      // sorted pairs per tile
  static constexpr int BN = 256;                      // weight rows per task
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * kStageBytesK;   // 16 KB of pairs
  static constexpr int B_BYTES = BN * kStageBytesK;   // 32 KB of weights
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // warpgroup 0: producer (warp 0), MMA issuer and TMEM owner (warp 1), two
  // idle warps; warpgroups 1-2: epilogue.  Launched at REGS registers per
  // thread, warpgroup 0 gives registers up and the epilogue takes them:
  // 128 * REGS_LOW + 256 * REGS_HIGH == 384 * REGS, so setmaxnreg.inc always
  // finds what it asks for (the launcher checks the compiled count is REGS).
  static constexpr int EPI_WARPS = 8;
  static constexpr int EPI_THREADS = EPI_WARPS * 32;
  static constexpr int THREADS = 128 + EPI_THREADS;
  static constexpr int REGS = 168, REGS_LOW = 104, REGS_HIGH = 200;
  static_assert(128 * REGS_LOW + 256 * REGS_HIGH == THREADS * REGS, "register split");
  static constexpr int COLS = 64;                     // columns of one half per epilogue thread
  // GEMM2: one 32-row x 32-column bf16 staging tile per epilogue warp
  static constexpr int STG_BYTES = EPI_WARPS * 32 * 32 * 2;
  // GEMM1: the two halves' amax of each pair, double-buffered by task
  static constexpr int AMAX_BYTES = 2 * 2 * BM * 4;
  // the operand scale blocks of the K blocks in flight
  static constexpr int SF_SLOTS = 8;
  static constexpr int SF_BYTES = SF_SLOTS * 512;
  static constexpr int TABLE_INTS = kMaxE + 8;
  static constexpr int SMEM = STAGES * STAGE_BYTES + STG_BYTES + AMAX_BYTES + SF_BYTES + 1024 + 3 * TABLE_INTS * 4 + 1024;
  static constexpr uint32_t IDESC = idesc_f8f6f4(FMT8_E4M3, FMT8_E4M3, BM, BN);
  static_assert(2 * BN <= 512, "two partials in TMEM");
  static_assert(SMEM <= 232448, "shared memory");
};

template <bool G1>
__global__ void __launch_bounds__(WCfg<G1>::THREADS, 1)
k_gemm_wide(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmT,
            const GemmParams p) {
  using C = WCfg<G1>;
  constexpr int KIND = G1 ? G1_F8 : G2_F8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  uint16_t* stg_all = reinterpret_cast<uint16_t*>(smem + C::STAGES * C::STAGE_BYTES);
  float* amax_sh = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES + C::STG_BYTES);
  uint8_t* sfring = smem + C::STAGES * C::STAGE_BYTES + C::STG_BYTES + C::AMAX_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sfring + C::SF_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;   // K-block partial full
  uint64_t* acce = accf + 2;            // ... and drained by the epilogue
  uint64_t* sfull = acce + 2;           // scale block landed
  uint64_t* sempty = sfull + C::SF_SLOTS;   // ... and read by every epilogue warp
  uint64_t* epibar = sempty + C::SF_SLOTS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(epibar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* tab = reinterpret_cast<int*>(sfring + C::SF_BYTES + 1024);
  const Tables tbl{tab, tab + C::TABLE_INTS, tab + 2 * C::TABLE_INTS};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&accf[b], 1); mbar_init(&acce[b], C::EPI_WARPS); }
    for (int b = 0; b < C::SF_SLOTS; ++b) { mbar_init(&sfull[b], 1); mbar_init(&sempty[b], C::EPI_WARPS); }
    mbar_init(epibar, C::EPI_THREADS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmT); }
  if (warp == 1) { tmem_alloc(tmem_holder, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  pdl_wait();  // inputs of this step are complete and visible
  pdl_launch_dependents();
  for (int i = threadIdx.x; i <= p.E; i += C::THREADS) {
    tab[i] = __ldcg(p.tiles + i);
    tab[C::TABLE_INTS + i] = __ldcg(p.offsets + i);
    tab[2 * C::TABLE_INTS + i] = i < p.E ? __ldcg(p.counts + i) : 0;
  }
  __syncthreads();

  const int total = tbl.tiles[p.E] * p.jn;
  const uint64_t deadline = globaltimer() + p.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    setmaxnreg_dec<C::REGS_LOW>();
    int stage = 0, kb_it = 0;
    uint32_t phase = 0;
    for (int idx = blockIdx.x; idx < total; idx += gridDim.x) {
      Task t;
      decode_task(p, tbl, idx, C::BM, G1, t);
      bool ok = true;
      int kfail = 0;
      for (int kst = t.k0; kst < t.k1; ++kst, ++kb_it) {
        if (!mbar_wait(&empty[stage], phase ^ 1, deadline, abort_flag)) { ok = false; kfail = kst; break; }
        const int slot = kb_it % C::SF_SLOTS;
        if (!mbar_wait(&sempty[slot], ((kb_it / C::SF_SLOTS) & 1) ^ 1, deadline, abort_flag)) {
          ok = false; kfail = kst; break;
        }
        if (lane == 0) {
          // the tile's operand scales of this K block, packed 512-byte block
          mbar_arrive_expect_tx(&sfull[slot], 512);
          bulk_load(sfring + slot * 512, p.bsf + ((size_t)t.tile * p.nchb + kst) * 512, 512, &sfull[slot]);
          uint8_t* sb = stages + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sb, &tmT, &full[stage], kst * kStageBytesK, t.row0);
          // GEMM1: gate rows j*128.., up rows I + j*128..; GEMM2: h-tiles 2j and
          // 2j + 1 (past H the copy fills zeros and the rows are not stored)
          const int r0 = G1 ? t.j * kTileW : 2 * t.j * kTileW;
          const int r1 = G1 ? p.I + t.j * kTileW : (2 * t.j + 1) * kTileW;
          tma_load_3d(sb + C::A_BYTES, &tmW, &full[stage], kst * kStageBytesK, r0, t.e);
          tma_load_3d(sb + C::A_BYTES + C::B_BYTES / 2, &tmW, &full[stage], kst * kStageBytesK, r1, t.e);
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      __syncwarp();
      if (!ok) {
        if (lane == 0) flag_timeout(p, abort_flag, KIND, W_PROD_EMPTY, kfail);
        const uint64_t until = globaltimer() + 2000000ull;   // copies in flight land first
        while (globaltimer() < until) { }
        break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    setmaxnreg_dec<C::REGS_LOW>();
    if (lane == 0) {
      int stage = 0, kb_it = 0, site = 0, kfail = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        Task t;
        decode_task(p, tbl, idx, C::BM, G1, t);
        for (int kst = t.k0; kst < t.k1; ++kst, ++kb_it) {
          if (!mbar_wait(&full[stage], phase, deadline, abort_flag)) { ok = false; site = W_MMA_FULL; kfail = kst; break; }
          const int pb = kb_it & 1;
          if (!mbar_wait(&acce[pb], ((kb_it >> 1) & 1) ^ 1, deadline, abort_flag)) {
            ok = false; site = W_MMA_PEMPTY; kfail = kst; break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(stages + stage * C::STAGE_BYTES), b_base = a_base + C::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f8f6f4(tmem + pb * C::BN, sdesc_sw128(a_base + ks * 32), sdesc_sw128(b_base + ks * 32), C::IDESC,
                       ks > 0);
          tc_commit(&empty[stage]);
          tc_commit(&accf[pb]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        flag_timeout(p, abort_flag, KIND, site, kfail);
        tc_commit(&accf[0]);   // drain this thread's tensor-core work before TMEM is released
        const uint64_t until = globaltimer() + 2000000ull;
        while (globaltimer() < until) { }
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    setmaxnreg_dec<C::REGS_LOW>();   // idle
  } else {
    // ------------------------------------------------------ epilogue
    setmaxnreg_inc<C::REGS_HIGH>();
    const int ew = warp - 4, q = warp & 3, half = ew >> 2;   // q: the warp's TMEM lane quarter
    const int row = 32 * q + lane;                           // pair inside the tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16);
    uint16_t* stg = stg_all + ew * 32 * 32;
    int tcount = 0, kb_it = 0, kfail = 0;
    bool ok = true;
    uint32_t epi_phase = 0;
    auto epi_bar = [&]() -> bool {
      mbar_arrive(epibar);
      const bool got = mbar_wait(epibar, epi_phase, deadline, abort_flag);
      epi_phase ^= 1;
      return got;
    };
    // the weights' block scales of a task, one per K block and half, spread
    // over the lanes (K block b in lane b % 32, register b / 32) a task ahead
    constexpr int SWR = 2;
    float swc[2][SWR], swn[2][SWR];
    const bool sw_in_regs = p.kst <= 32 * SWR;
    auto sw_ptr = [&](const Task& tt, int a, int kb) -> const float* {
      if (G1) return p.sfa_f32 + ((size_t)tt.e * (2 * p.I / 128) + (a ? p.I / 128 : 0) + tt.j) * (p.H / 128) + kb;
      return p.sfa_f32 + ((size_t)tt.e * (p.H / 128) + min(2 * tt.j + a, p.H / 128 - 1)) * (p.I / 128) + kb;
    };
    auto load_sw = [&](int idx, float (&dst)[2][SWR]) {
      if (!sw_in_regs || idx >= total) return;
      Task tn;
      decode_task(p, tbl, idx, C::BM, G1, tn);
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int r = 0; r < SWR; ++r) {
          const int kb = tn.k0 + lane + 32 * r;
          dst[a][r] = kb < tn.k1 ? __ldg(sw_ptr(tn, a, kb)) : 0.0f;
        }
    };
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int r = 0; r < SWR; ++r) { swc[a][r] = 0.0f; swn[a][r] = 0.0f; }
    load_sw(blockIdx.x, swn);

    for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x, ++tcount) {
      Task t;
      decode_task(p, tbl, idx, C::BM, G1, t);
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int r = 0; r < SWR; ++r) swc[a][r] = swn[a][r];
      load_sw(idx + (int)gridDim.x, swn);
      const float wpair = (!G1 && row < t.valid) ? __ldcg(p.sorted_w + t.row0 + row) : 0.0f;

      float acc[2][C::COLS];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int i = 0; i < C::COLS; ++i) acc[a][i] = 0.0f;
      for (int kst = t.k0; kst < t.k1; ++kst, ++kb_it) {
        // the pair's operand scale: E8M0 byte of the packed block (row r of a
        // tile at word 4 * (r % 32) + r / 32), from the scale ring
        const int slot = kb_it % C::SF_SLOTS;
        if (!mbar_wait(&sfull[slot], (kb_it / C::SF_SLOTS) & 1, deadline, abort_flag)) { ok = false; kfail = kst; break; }
        const uint32_t xw = reinterpret_cast<const uint32_t*>(sfring + slot * 512)[4 * lane + q];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[slot]);
        const float xsc = __uint_as_float((xw & 0xFFu) << 23);   // 2^(byte - 127)
        float f[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int kq = kst - t.k0;
          const float sw = sw_in_regs ? __shfl_sync(0xFFFFFFFFu, (kq >> 5) ? swc[a][1] : swc[a][0], kq & 31)
                                      : __ldg(sw_ptr(t, a, kst));
          f[a] = sw * xsc;
        }
        const int pb = kb_it & 1;
        if (!mbar_wait(&accf[pb], (kb_it >> 1) & 1, deadline, abort_flag)) { ok = false; kfail = kst; break; }
        tc_fence_after();
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int c = 0; c < C::COLS / 32; ++c) {
            float v[32];
            tmem_ld32(tl + pb * C::BN + a * (C::BN / 2) + half * C::COLS + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; i += 2) fma2(acc[a][c * 32 + i], acc[a][c * 32 + i + 1], f[a], v[i], v[i + 1]);
          }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[pb]);
      }
      if (!ok) break;

      if (G1) {
        // SwiGLU, then mid quantized once per (pair, 128-block): power-of-two
        // scale from the amax over both halves, E4M3
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < C::COLS; ++i) {
          acc[0][i] = silu_mul(acc[0][i], acc[1][i]);
          amax = fmaxf(amax, fabsf(acc[0][i]));
        }
        float* ash = amax_sh + (tcount & 1) * 2 * C::BM;
        ash[half * C::BM + row] = amax;
        if (!epi_bar()) { ok = false; break; }
        amax = fmaxf(amax, ash[(1 - half) * C::BM + row]);
        const int ke = pow2_e4m3_exp(amax);
        const float inv = exp2i(-ke);
        if (row < t.valid) {
          const size_t r = (size_t)(t.row0 + row);
          uint4* dst = reinterpret_cast<uint4*>(p.midq + r * p.I + t.j * kTileW + half * C::COLS);
#pragma unroll
          for (int c = 0; c < C::COLS / 16; ++c) {
            const float* m = acc[0] + c * 16;
            dst[c] = make_uint4(cvt_e4m3x4(m[0] * inv, m[1] * inv, m[2] * inv, m[3] * inv),
                                cvt_e4m3x4(m[4] * inv, m[5] * inv, m[6] * inv, m[7] * inv),
                                cvt_e4m3x4(m[8] * inv, m[9] * inv, m[10] * inv, m[11] * inv),
                                cvt_e4m3x4(m[12] * inv, m[13] * inv, m[14] * inv, m[15] * inv));
          }
          if (half == 0) p.midqs[r * (p.I / 128) + t.j] = exp2i(ke);
        }
        // GEMM2's operand scale for this pair and 128-block, packed like the token scales
        if (half == 0) p.bsf_out[((size_t)t.tile * (p.I / 128) + t.j) * 128 + 4 * lane + q] = rep4((uint32_t)(ke + 127));
      } else {
        // bf16(w * y): the warp's 32 pairs x 32 columns at a time through its
        // staging tile (16-byte chunks of a row XOR-rotated by (row / 2) % 4),
        // then 16-byte stores, 8 rows of 64 bytes per instruction
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int ht = 2 * t.j + a;
          if (ht * kTileW >= p.H) break;
#pragma unroll
          for (int cc = 0; cc < C::COLS / 32; ++cc) {
            __syncwarp();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const float* v = acc[a] + cc * 32 + ch * 8;
              const uint4 w4 = make_uint4(bf16x2_bits(wpair * v[0], wpair * v[1]), bf16x2_bits(wpair * v[2], wpair * v[3]),
                                          bf16x2_bits(wpair * v[4], wpair * v[5]), bf16x2_bits(wpair * v[6], wpair * v[7]));
              *reinterpret_cast<uint4*>(stg + lane * 32 + ((ch ^ ((lane >> 1) & 3)) * 8)) = w4;
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = 8 * i + (lane >> 2), ch = lane & 3;
              const uint4 w4 = *reinterpret_cast<const uint4*>(stg + r * 32 + ((ch ^ ((r >> 1) & 3)) * 8));
              if (32 * q + r < t.valid)
                *reinterpret_cast<uint4*>(p.yw + (size_t)(t.row0 + 32 * q + r) * p.H + ht * kTileW + half * C::COLS +
                                          cc * 32 + ch * 8) = w4;
            }
          }
        }
      }
    }
    if (!ok && lane == 0) flag_timeout(p, abort_flag, KIND, W_EPI_ACCF, kfail);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host-side launch helpers (instantiations used by the API).
template <int KIND, int NT, int STAGES>
static cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, int grid,
                              cudaStream_t st) {
  using C = GCfg<KIND, NT, STAGES>;
  auto kern = k_gemm<KIND, NT, STAGES>;
  static bool attr_set[64] = {false};   // per device; set outside any stream capture on first use
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, b, p);
}

template <bool G1>
static cudaError_t launch_wide(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, int grid,
                               cudaStream_t st) {
  using C = WCfg<G1>;
  auto kern = k_gemm_wide<G1>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    // the register split inside the kernel assumes exactly C::REGS at launch
    cudaFuncAttributes fa;
    cudaError_t err = cudaFuncGetAttributes(&fa, kern);
    if (err != cudaSuccess) return err;
    if (fa.numRegs != C::REGS) return cudaErrorInvalidKernelImage;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, b, p);
}

cudaError_t launch_gemm1(int wfmt, int nt, const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p,
                         int grid, cudaStream_t st) {
  if (wfmt == MOE_W_MXFP4) {
    switch (nt) {
      case 16: return launch_one<G1_MX, 16, 5>(a, b, p, grid, st);
      case 32: return launch_one<G1_MX, 32, 5>(a, b, p, grid, st);
      case 64: return launch_one<G1_MX, 64, 4>(a, b, p, grid, st);
    }
  } else {
    switch (nt) {
      case 16: return launch_one<G1_F8, 16, 5>(a, b, p, grid, st);
      case 32: return launch_one<G1_F8, 32, 5>(a, b, p, grid, st);
      case 64: return launch_one<G1_F8, 64, 4>(a, b, p, grid, st);
      case 128: return p.split == 1 ? launch_wide<true>(a, b, p, grid, st) : cudaErrorInvalidValue;
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm2(int wfmt, int nt, const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p,
                         int grid, cudaStream_t st) {
  if (wfmt == MOE_W_MXFP4) {
    switch (nt) {
      case 16: return launch_one<G2_MX, 16, 4>(a, b, p, grid, st);
      case 32: return launch_one<G2_MX, 32, 4>(a, b, p, grid, st);
      case 64: return launch_one<G2_MX, 64, 4>(a, b, p, grid, st);
    }
  } else {
    switch (nt) {
      case 16: return launch_one<G2_F8, 16, 4>(a, b, p, grid, st);
      case 32: return launch_one<G2_F8, 32, 4>(a, b, p, grid, st);
      case 64: return launch_one<G2_F8, 64, 4>(a, b, p, grid, st);
      case 128: return launch_wide<false>(a, b, p, grid, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
