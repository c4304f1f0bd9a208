/* fp64 CPU oracle of the routed block-quantised MoE layer (test infrastructure;
 * see oracle.c for what it computes and the passages it follows). */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

enum { ORACLE_Q8_0 = 1, ORACLE_Q5_1 = 2, ORACLE_IQ4_NL = 3, ORACLE_NVFP4 = 4, ORACLE_Q5_0 = 5 };

typedef struct {
    int n_experts, hidden, inter, has_shared;
    int fmt_gate_up, fmt_down;
    const uint8_t *gate_up;        /* canonical blocks, per expert [2I rows x H] */
    const uint8_t *down;           /* canonical blocks, per expert [H rows x I]  */
    const double *gate_up_scale;   /* NVFP4 matrix scales per expert (shared last), else NULL */
    const double *down_scale;
    const int8_t *table;           /* IQ4_NL 16-entry table, else NULL */
} oracle_desc;

double oracle_fp16(uint16_t u);
double oracle_bf16(uint16_t u);
double oracle_e4m3(int c);
double oracle_e2m1(int c);
int64_t oracle_row_bytes(int fmt, int64_t cols);
int oracle_decode_row(int fmt, const uint8_t *row, int64_t cols, const int8_t *table,
                      double tensor_scale, double *out);
void oracle_route_token(const double *x, const uint16_t *wr, int H, int E, int k, int32_t *idx,
                        double *gate, double *logits);
void oracle_route(const double *x, const uint16_t *wr, int T, int H, int E, int k, int32_t *idx,
                  double *gate, double *logits);
void oracle_act_quant_nvfp4(const double *in, int64_t n, double *out);
int oracle_expert(const oracle_desc *d, int e, const double *x, double *y, int act_quant);
int oracle_layer(const oracle_desc *d, const double *x, const uint16_t *wr, int T, int k,
                 double *out, int32_t *idx_out, double *gate_out, int act_quant);
int oracle_threads(void);
void oracle_set_threads(int n);
#endif
