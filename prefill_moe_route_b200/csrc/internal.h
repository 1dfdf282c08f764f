// internal.h -- host/device shared definitions of libmoe_b200: kernel
// parameter blocks, the workspace plan and the tile configuration chosen per
// shape.  Not part of the public ABI (include/moe_b200.h is).
#pragma once
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kMaxE = 512;
constexpr int kMaxTopk = 16;
constexpr int kTileW = 128;        // weight rows per MMA (M of the instruction)
constexpr int kStageBytesK = 128;  // bytes of one operand row per pipeline stage

// Device status word bits (workspace status[0]).
enum : int32_t { ST_TIMEOUT = 1, ST_BAD_TASK = 2, ST_BAD_INPUT = 4 };

// One expert-major plan shared by the kernels of a call.
struct Plan {
  int M, H, I, E, topk, wfmt;
  float routed_scale;
  int P;        // M * topk pairs
  int nt1;      // token (pair) rows per GEMM1 tile: MMA N
  int nt2;      // token rows per GEMM2 tile
  int split1;   // K splits of GEMM1 (small M)
  int kst1;     // GEMM1 pipeline stages over K (H / elements per stage)
  int kst2;     // GEMM2 stages over K (I / 128)
  int j1;       // I / 128 n-tiles of GEMM1 (each a gate tile + an up tile)
  int ht2;      // H / 128 h-tiles of GEMM2
  int groups1;  // upper bound of (expert, token tile, n-tile) groups for split-K
  // workspace offsets (bytes)
  size_t o_status, o_ids, o_w, o_counts, o_offsets, o_sorted, o_inv, o_tiles1, o_tiles2;
  size_t o_xq, o_xs, o_midq, o_midqs, o_y, o_part, o_cnt1, o_sync, o_flags, o_midsf, o_midt, o_xpart, o_xflag, total;
  size_t o_chunk;     // [nchunks][E] chunk counts of the sort (zero between calls)
  size_t o_sortw;     // [P] routing weight of each sorted pair
  size_t o_bsf1, o_bsf2;   // packed operand scales of GEMM1 / GEMM2 [tiles][K/128][512 B]
  size_t o_xg;        // GEMM1's operand rows in sorted-pair order
  int tiles_max;      // upper bound of token tiles over all experts
  int chunk_tokens, nchunks;
  bool small;   // single-launch path (decode-sized MXFP4 calls)
};

// Filled by the host from a shape; returns MOE_OK or an error code.
int make_plan(const moe_shape_t& s, int num_sms, Plan* p);

// Parameters of the route / activation-quant / align kernel.
struct RouteParams {
  const float* logits;      // null when the caller routed (ids_in / w_in)
  const float* bias;        // may be null
  const int32_t* ids_in;    // caller's selection [M][topk], or null
  const float* w_in;        // caller's weights [M][topk], or null
  const uint16_t* x;        // may be null (routing only)
  int32_t* topk_ids;
  float* topk_w;
  uint8_t* xq;
  void* xs;
  int32_t* status;          // [0] status word, [1] arrival counter
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_pairs;
  int32_t* inv;
  float* sorted_w;          // [P] routing weight of each sorted pair
  uint32_t* bsf;            // GEMM1's operand scales packed per (token tile, 128-column chunk): 512 B blocks
  uint8_t* xg;              // GEMM1's operand rows in sorted-pair order [P][quantized row bytes]
  int32_t* tiles1;          // [E+1] prefix of ceil(count/nt1)
  int32_t* tiles2;          // [E+1] prefix of ceil(count/nt2)
  int32_t* chunk_cnt;       // [nchunks][E] pairs per (chunk, expert), then their prefixes; zero between calls
  int chunk_tokens;         // tokens per chunk of the sort
  int chunk_pairs;          // chunk_tokens * topk
  int nchunks;
  int M, E, topk, H, wfmt, nt1, nt2;
  float routed_scale;
  int do_align;
};

struct GemmParams {
  // routing products
  const int32_t* offsets;
  const int32_t* counts;
  const int32_t* sorted_pairs;
  const int32_t* tiles;     // tiles1 (GEMM1) or tiles2 (GEMM2)
  // scales
  const uint8_t* sfa_u8;    // MXFP4 weight scales (E8M0), packed 512-byte blocks
  const float* sfa_f32;     // FP8 weight block scales
  const uint8_t* bsf;       // operand (token / mid) scales, packed: [token tile][K/128][512 B]
  int nchb;                 // 128-column chunks of K in bsf (GEMM1: H/128, GEMM2: I/128)
  uint32_t* bsf_out;        // GEMM1: GEMM2's operand scales, packed the same way
  // outputs
  uint8_t* midq;
  float* midqs;
  const float* sorted_w;    // GEMM2: routing weight of each sorted pair
  uint16_t* yw;             // GEMM2 output: bf16(w * y) [P][H], rows in sorted order
  float* part;              // split-K partials
  int32_t* cnt;             // split-K arrival counters
  int32_t* status;
  int M, H, I, E, topk, P;
  int kst;                  // stages over the whole K
  int split;                // K splits
  int jn;                   // n-tiles (GEMM1: I/128) or h-tiles (GEMM2: H/128)
  uint64_t timeout_ns;
};

// Parameters of the single-launch small-batch kernel (small.cu).
struct SmallParams {
  const uint16_t* x;
  const float* logits;      // null when the caller routed (ids_in / w_in)
  const float* bias;        // may be null
  const int32_t* ids_in;    // caller's selection [M][topk], or null
  const float* w_in;        // caller's weights [M][topk], or null
  const uint8_t* w2;        // w2 E2M1 codes [E][H][I/2] (L2 prefetch only; the MMA reads it by TMA)
  const uint8_t* s13;       // w13 E8M0 scales [E][2I][H/32]
  const uint8_t* s2;        // w2 E8M0 scales [E][H][I/32]
  uint16_t* out;
  float* out_f32;           // non-null: the call's fp32 sum [M][H] instead of bf16 out (a TP rank's partial)
  int32_t* status;
  int32_t* sync;            // [0] completed-call epoch, [1] exit counter
  int32_t* flags;           // [E][16] epoch of each published (expert, n-tile) of mid
  int32_t* topk_ids;
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_pairs;
  int32_t* inv;
  uint8_t* midq;
  float* midqs;
  uint32_t* midsf;          // [E][I/128][64] mid scales as the MMA's B scale-factor rows (row = token, 16-byte stride)
  uint8_t* midt;            // [E][16][I] mid E4M3 codes, row = token (GEMM2's B operand)
  float* xpart;             // [H/128][128][16] partner halves of split h-tiles
  int32_t* xflag;           // [H/128] epoch of each published partner half
  int M, H, I, E, topk;
  float routed_scale;
  uint64_t timeout_ns;
  int test_withhold;        // test knob: leave the first mid flag of the call unpublished
};

struct CombineParams {
  const uint16_t* yw;       // bf16(w * y) [P][H], rows in sorted order
  const int32_t* inv;
  uint16_t* out;
  float* out_f32;           // non-null: fp32 sums instead of bf16 out (a TP rank's partial)
  int M, H, topk;
};

}  // namespace moe
