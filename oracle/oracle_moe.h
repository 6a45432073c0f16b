/*
 * oracle_moe.h -- declarations of the fp64 CPU parity oracle.
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, bench CPU baseline).
 * Nothing here is shared with the CUDA library.
 */
#ifndef ORACLE_MOE_H
#define ORACLE_MOE_H
#include <stddef.h>
#include <stdint.h>

#define ORC_QBLOCK 32
#define ORC_QBLOCK_BYTES 10

double orc_half_to_double(uint16_t h);
double orc_bf16_to_double(uint16_t b);
uint16_t orc_double_to_bf16(double v);
void orc_double_to_bf16_array(size_t n, const double *v, uint16_t *out);
void orc_dequant_block(const uint8_t *blk, double *w);
void orc_dequant_matrix(const uint8_t *blocks, int rows, int cols, double *W);
size_t orc_expert_bytes(int hidden, int inter);
double orc_silu(double z);
void orc_expert_forward(int hidden, int inter, const uint8_t *expert, const double *x, double *y);
void orc_topk_one(const double *logits, int n_experts, int top_k, int32_t *idx, double *w, double *gap);
void orc_logits_one(int hidden, int n_experts, const double *x, const float *router_w, const float *router_b,
                    double *logits);
int orc_route(int hidden, int n_experts, int top_k, int tokens, const uint16_t *x_bf16, const float *router_w,
              const float *router_b, int32_t *idx, double *w, double *gap, double *logits_out);
int orc_layer(int hidden, int inter, int n_experts, int top_k, int tokens, const uint16_t *x_bf16,
              const float *router_w, const float *router_b, const uint8_t *experts, const uint8_t *shared,
              const int32_t *forced_idx, double *y, int32_t *idx_out, double *w_out, double *gap_out);
void orc_rmsnorm(int n, const double *v, double eps, double *out);
int orc_stack(int hidden, int inter, int n_experts, int top_k, int n_layers, int tokens, const uint16_t *x_bf16,
              const double *resid_in, const float *const *router_w, const float *const *router_b, const uint8_t *const *experts,
              const uint8_t *const *shared, double eps, const int32_t *follow_idx, double tie_gap, double *resid,
              int32_t *idx_out, double *gap_out, int *n_followed, int *n_mismatch);
int orc_num_threads(void);
void orc_set_num_threads(int n);
#endif
