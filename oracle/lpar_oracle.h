/*
 * lpar_oracle.h -- declarations of the CPU oracle (test infrastructure only).
 *
 * Only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * may use this.  It is independent of the CUDA library: no shared header,
 * constant or helper.  Codec numbers are the oracle's own.
 *
 * All buffers are host memory owned by the caller.  Sizes are in elements
 * unless named *_bytes.  n must be a multiple of ORC_TILE_ELEMS.
 */
#ifndef LPAR_ORACLE_H
#define LPAR_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_BF16 = 0, ORC_FP8 = 1, ORC_INT4 = 2, ORC_INT3 = 3, ORC_MXFP4 = 4 };
enum { ORC_BLOCK = 32, ORC_TILE_ELEMS = 2048, ORC_BLOCKS_PER_TILE = 64, ORC_MAX_RANKS = 8 };

/* number formats */
float    orc_bf16_to_f32(uint16_t h);
uint16_t orc_f32_to_bf16_rne(float x);
uint16_t orc_f32_to_f16_rne(float x);
float    orc_f16_to_f32(uint16_t h);
float    orc_e4m3_to_f32(uint8_t e);
uint8_t  orc_f32_to_e4m3_rne_satfinite(float x);
float    orc_e2m1_to_f32(uint8_t c);
uint8_t  orc_e2m1_rne_satfinite(double y);
double   orc_e8m0_to_f64(uint8_t code);

/* geometry */
size_t orc_tile_bytes(int codec);
size_t orc_wire_bytes(int codec, size_t n);

/* one 32-element block */
void  orc_quant_block_int(const float *x, int bits, uint16_t *scale_bits, uint8_t *codes);
float orc_dequant_int(uint8_t code, int bits, uint16_t scale_bits);
void  orc_quant_block_fp8(const float *x, float *scale, uint8_t *codes);
float orc_dequant_fp8(uint8_t code, float scale);
void  orc_quant_block_mxfp4(const float *x, uint8_t *scale_code, uint8_t *codes);
float orc_dequant_mxfp4(uint8_t code, uint8_t scale_code);

/* one 2048-element tile */
void    orc_quant_tile(const float *x, int codec, uint8_t *tile);
uint8_t orc_tile_code(const uint8_t *tile, int codec, int i);
void    orc_dequant_tile(const uint8_t *tile, int codec, float *v);

/* stages and the whole collective */
void orc_quantize(const uint16_t *in_bf16, size_t n, int codec, uint8_t *wire);
void orc_reduce(const uint8_t *const *wires, int N, size_t tile_begin, size_t tile_count,
                int codec, uint8_t *wire_out);
void orc_decode(const uint8_t *wire, size_t n, int codec, uint16_t *out_bf16);
int  orc_allreduce(const uint16_t *const *in_bf16, int N, size_t n, int codec,
                   uint16_t *const *out_bf16, size_t min_quant_bytes);

/* standalone collectives and the one-shot all-reduce (return the codec used, or -1) */
int orc_reduce_scatter(const uint16_t *const *in_bf16, int N, size_t n, int codec,
                       uint16_t *const *out_bf16, size_t min_quant_bytes);
int orc_allreduce_oneshot(const uint16_t *const *in_bf16, int N, size_t n, int codec,
                          uint16_t *const *out_bf16, size_t min_quant_bytes);
int orc_all_gather(const uint16_t *const *in_bf16, int N, size_t m, int codec,
                   uint16_t *const *out_bf16, size_t min_quant_bytes);
int orc_all_to_all(const uint16_t *const *in_bf16, int N, size_t m, int codec,
                   uint16_t *const *out_bf16, size_t min_quant_bytes);

/* the all-reduce of binary32 messages (binary32 results; codec 0 = uncompressed) */
int orc_allreduce_f32(const float *const *in_f32, int N, size_t n, int codec,
                      float *const *out_f32, size_t min_quant_bytes);

#ifdef __cplusplus
}
#endif
#endif
