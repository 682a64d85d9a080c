/*
 * oracle.h -- declarations of the CPU oracle (test infrastructure only).
 * The CUDA library never includes this header and the oracle never includes
 * the library's; see oracle.c for the definitions and their sources.
 */
#ifndef KVQ_ORACLE_H
#define KVQ_ORACLE_H

#include <stdint.h>

#define ORACLE_RN 0 /* round to nearest, ties to even */
#define ORACLE_RD 1 /* round toward -infinity */
#define ORACLE_RU 2 /* round toward +infinity */

uint16_t oracle_f32_to_f16(float v, int mode);
void oracle_f32_to_f16_array(const float *v, int64_t n, int mode, uint16_t *out);
float oracle_f16_to_f32(uint16_t h);
uint16_t oracle_f32_to_bf16_rn(float v);
void oracle_f32_to_bf16_rn_array(const float *v, int64_t n, uint16_t *out);
float oracle_bf16_to_f32(uint16_t b);

void oracle_fwht_f32(float *x, int n);
void oracle_rotate_blocks_f32(float *x, int64_t n_vec, int D, int hb);
void oracle_fwht_f64(double *x, int n);
void oracle_rotate_blocks_f64(double *x, int64_t n_vec, int D, int hb);

void oracle_quantize_group(const float *x, int n, int stride, int bits,
                           uint16_t *s_out, uint16_t *z_out, uint8_t *q_out,
                           int q_stride);
void oracle_quantize_group_hybrid(const float *x, int n, int stride, int bits,
                                  uint16_t *s_out, uint16_t *z_out,
                                  uint8_t *q_out, int q_stride);
void oracle_pack_codes(const uint8_t *q, int n, int bits, uint8_t *out);
void oracle_unpack_codes(const uint8_t *packed, int n, int bits, uint8_t *q);
void oracle_quantize_tokens(const float *x, int64_t n_vec, int D, int hb,
                            int G, int bits, int hybrid, uint8_t *codes,
                            uint16_t *sz);
void oracle_quantize_channel_block(const float *x, int R, int D, int bits,
                                   int hybrid, uint8_t *codes, uint16_t *sz);
void oracle_dequant_tokens(const uint8_t *codes, const uint16_t *sz,
                           int64_t n_vec, int D, int G, int bits, double *out);
void oracle_dequant_channel_block(const uint8_t *codes, const uint16_t *sz,
                                  int R, int D, int bits, double *out);

void oracle_attention(const double *q, int n_q, const double *k,
                      const double *v, int64_t T, int D, double scale,
                      double *out);

void oracle_dequant_x_bf16(const uint8_t *codes, const uint16_t *sz,
                           int64_t n_tok, int hidden, int G, int bits,
                           float *xhat);
void oracle_matmul_nt(const float *a, const float *w, int64_t M, int N, int K,
                      double *out);
void oracle_rope(double *x, const int64_t *pos, int64_t M, int H, int D,
                 double theta);

#endif
