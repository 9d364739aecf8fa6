/*
 * msa_oracle.h — CPU oracle for MSA decode over an NVFP4 KV cache.
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the
 * benchmark).  Independent of the CUDA path: shares no header with it.
 * See msa_oracle.c for the definitions and the passages they follow.
 */
#ifndef MSA_ORACLE_H
#define MSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* An NVFP4 cache: planes data [B][heads][lmax][dim/2] and scale
 * [B][heads][lmax][dim/16] (E4M3), one fp32 tensor scale. */
typedef struct orc_nvfp4 {
    const uint8_t* data;
    const uint8_t* scale;
    float tensor_scale;
    int heads;
    int dim;
    int64_t lmax;
} orc_nvfp4;

double orc_e2m1_value(uint8_t code);
double orc_e4m3_value(uint8_t code);
uint8_t orc_e4m3_encode(float x);
uint8_t orc_e2m1_encode(float x);

float orc_tensor_scale(const float* x, int64_t n);
void orc_nvfp4_encode(const float* x, int64_t nvec, int dim, float s_tensor,
                      uint8_t* data, uint8_t* scale);
void orc_nvfp4_decode(const uint8_t* data, const uint8_t* scale, int64_t nvec, int dim,
                      float s_tensor, float* out);

void orc_index(int B, int Tq, int HI, int DI, const int32_t* seq_lens,
               const float* q_idx, const float* w_idx, const orc_nvfp4* ik,
               int pool_mode, double* token_scores, double* block_scores);
void orc_select(int B, int Tq, int64_t nbmax, const int32_t* seq_lens,
                const double* block_scores, int32_t* sel);
void orc_attend(int B, int Tq, int Hq, int Hkv, int D, const int32_t* seq_lens,
                const float* q, const orc_nvfp4* k, const orc_nvfp4* v,
                const int32_t* sel, double scale, double* out, double* lse);
int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
