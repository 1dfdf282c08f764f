/*
 * moe_oracle.h -- plain CPU oracle for the quantized routed-expert MoE call.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code with the CUDA path (prefill_moe_route_b200/csrc) and must never be
 * linked into it.
 *
 * What it computes (one MoE layer call, per token t, slot j, expert e):
 *   route   s_e = sigmoid(l_e); top-k of s_e + b_e (ties -> lower expert ID);
 *           w_j = s_j / sum_j s_j * routed_scale
 *           ("glm53: Quantize each mid block ...", commit 3 message: top-8
 *            rounds, a tied round broken by expert ID)
 *   align   pairs p = t*k + j stably sorted by expert
 *           ("glm53_flash: score a verify request's index tiles once",
 *            commit message: expert-major MoE above 8 rows)
 *   quant   x -> MXFP4 (OCP E2M1 + E8M0 per 32) for the MXFP4 weight format,
 *           x -> E4M3 with a power-of-two scale per 128 for block FP8
 *           ("IQ2R: load GLM-5.3 packed MoE checkpoints", MXFP4 arm is A4W4)
 *   GEMM1   g = deq(xq) . deq(w13[e])^T         (fp64 accumulation)
 *   SwiGLU  mid = silu(g[:I]) * g[I:]           (rows [0,I) gate, [I,2I) up)
 *   midq    per (pair, 128-block of I): power-of-two scale, E4M3 codes
 *           ("glm53: FP8 mid hand-off", Modifications table row 1)
 *   GEMM2   y = deq(midq) . deq(w2[e])^T        (fp64 accumulation)
 *   combine out[t] = sum_j w_j * y[t,j]         (fp64, j ascending)
 *
 * Parity pins: every function here is checked by tests/test_oracle_*.py
 * against closed forms, brute force on tiny inputs, literal values of the
 * OCP MX v1.0 / OCP FP8 specifications (tests/golden/), invariants and the
 * mid hand-off sizes printed on the "FP8 mid hand-off" page.  End-to-end
 * numeric parity with the pages' own system is "parity unpinned": the pages
 * print no MoE input/output example.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_W_MXFP4 = 1, ORC_W_FP8_BLOCK128 = 2 };

typedef struct {
  int32_t M, H, I, E, topk;
  float routed_scale;
  int32_t wfmt;
} orc_shape_t;

/* ---- codecs (OCP MX v1.0; OCP 8-bit floating point, E4M3 "FN" variant) */
double  orc_e2m1_value(uint8_t code);      /* low 4 bits used            */
uint8_t orc_e2m1_encode(double v);         /* RNE on the grid, sat +-6   */
double  orc_e4m3_value(uint8_t code);      /* NaN for 0x7F / 0xFF        */
uint8_t orc_e4m3_encode(double v);         /* RNE, saturate to +-448     */
double  orc_e8m0_value(uint8_t code);      /* 2^(code-127), NaN for 0xFF */
uint16_t orc_bf16_encode(float v);         /* RNE                        */
float   orc_bf16_value(uint16_t b);

/* MX shared-scale rule for E2M1 blocks: X = 2^(floor(log2 amax) - 2),
 * exponent clamped to [-127, 127]; returns the E8M0 code (0 for amax = 0). */
uint8_t orc_mx_scale_code(float amax);
/* Power-of-two E4M3 scale: the smallest 2^k (k in [-126, 127]) with
 * amax <= 448 * 2^k; 1.0 for amax = 0.                                     */
float   orc_pow2_scale_e4m3(float amax);

/* MXFP4 quantization of `rows` rows of K fp32 values (K % 32 == 0).
 * packed: rows*K/2 bytes, element 2i in bits 3:0, 2i+1 in bits 7:4.
 * scales: rows*K/32 E8M0 codes.                                           */
void orc_quant_mxfp4(const float* w, int64_t rows, int32_t K,
                     uint8_t* packed, uint8_t* scales);
/* 128x128 block FP8 of a [rows, K] matrix: scale = amax/448 (fp32), 1 when
 * amax = 0; q = E4M3(w / scale) with the division in fp32.
 * scales: [rows/128][K/128] fp32.                                          */
void orc_quant_fp8_block128(const float* w, int32_t rows, int32_t K,
                            uint8_t* q, float* scales);
/* E4M3 with a power-of-two scale per 128 consecutive values (K % 128 == 0).
 * scales: K/128 fp32 values.                                               */
void orc_quant_fp8_pow2_row(const float* v, int32_t K, uint8_t* q, float* scales);

/* ---- routing sigmoid, specified to the operation so both sides agree:
 * exp via Cody-Waite reduction n = rint(x*log2e), r = (x - n*C1) - n*C2,
 * degree-7 Taylor polynomial in Horner form, times 2^n; x clamped to
 * [-87, 88]; every operation one fp32 round-to-nearest step.               */
float orc_exp_spec(float x);
float orc_sigmoid_spec(float l);

void orc_route(int32_t M, int32_t E, int32_t k, const float* logits,
               const float* bias /* nullable */, float routed_scale,
               int32_t* topk_ids, float* topk_w);

/* Stable counting sort of the M*k pairs by expert.
 * counts[E], offsets[E+1], sorted_pairs[M*k] (pair ids), inv[M*k]. */
void orc_align(int32_t M, int32_t k, int32_t E, const int32_t* topk_ids,
               int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
               int32_t* inv);

/* Quantize one activation row (bf16 bits) the way the format asks.
 * MXFP4: q = H/2 packed bytes, s = H/32 E8M0 codes (uint8).
 * FP8:   q = H E4M3 codes,     s = H/128 fp32 scales.                      */
void orc_quant_act_row(int32_t wfmt, const uint16_t* x_row, int32_t H,
                       uint8_t* q, void* s);

/* Forward for a subset of tokens (all tokens if toks == NULL, ntok = M).
 * Uses the caller's routing (topk_ids, topk_w) so the GEMM part can be
 * checked on its own.  Weights are quantized tensors:
 *   MXFP4: w13 [E][2I][H/2] + s13 [E][2I][H/32] u8, w2 [E][H][I/2] + s2 [E][H][I/32] u8
 *   FP8:   w13 [E][2I][H]   + s13 [E][2I/128][H/128] f32, w2 [E][H][I] + s2 [E][H/128][I/128] f32
 * Outputs for the n-th listed token (any may be NULL):
 *   midq  [ntok*k][I] E4M3 codes, pair order (t, j)
 *   midqs [ntok*k][I/128] fp32 power-of-two scales
 *   ref   [ntok][H] fp64 combine result; out [ntok][H] bf16 bits.
 * Returns 0, or -1 on a bad argument.                                      */
int orc_forward_tokens(const orc_shape_t* sh, const uint16_t* x,
                       const int32_t* topk_ids, const float* topk_w,
                       const uint8_t* w13, const void* s13,
                       const uint8_t* w2, const void* s2,
                       int32_t ntok, const int32_t* toks,
                       uint8_t* midq, float* midqs, double* ref,
                       uint16_t* out);

/* OpenMP thread count of the oracle's loops (timing only); returns the
 * previous count, n <= 0 leaves it unchanged.                             */
int orc_set_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
