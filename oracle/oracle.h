/* CPU oracle for paged decode attention (test infrastructure only). */
#ifndef PKV_ORACLE_H
#define PKV_ORACLE_H
#include <stdint.h>

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_E4M3 = 2, ORC_E5M2 = 3, ORC_INT8 = 4 };
enum { ORC_OK = 0, ORC_ERR_SHAPE = 1, ORC_ERR_DTYPE = 2, ORC_ERR_INDEX = 3, ORC_ERR_ALLOC = 4 };

double orc_e4m3_value(uint8_t code);
uint8_t orc_e4m3_encode(float x);
void orc_e4m3_encode_array(const float* x, uint8_t* codes, int64_t n);
double orc_e5m2_value(uint8_t code);
uint8_t orc_e5m2_encode(float x);
void orc_e5m2_encode_array(const float* x, uint8_t* codes, int64_t n);
int8_t orc_int8_encode(float x);

/* out: [len(seqs) or num_seqs][q_len][num_heads][head_dim] doubles, rows in the order
 * of `seqs` (all sequences when seqs == NULL); q: [num_seqs][q_len][num_heads][head_dim].
 * Query j of sequence s sits at position seq_lens[s] - q_len + j and attends the
 * tokens up to and including it (q_len = 1: plain decode). */
int orc_paged_decode(double* out,
                     const void* q, int q_dtype,
                     const void* k_cache, const void* v_cache, int kv_dtype,
                     const int32_t* block_tables, const int32_t* seq_lens,
                     int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                     int block_size, int max_blocks_per_seq, int num_blocks,
                     double scale, double k_scale, double v_scale,
                     const int32_t* seqs, int n_seqs, int q_len,
                     const float* k_head_scales, const float* v_head_scales);

/* orc_paged_decode that also writes, when lse != NULL, the natural log of each query
 * row's softmax denominator, log sum_t exp(scale * q . K_t) ([rows][q_len][num_heads];
 * -inf for a row that sees no token): what two disjoint parts of a sequence need to
 * be combined into the attention over both. */
int orc_paged_decode_lse(double* out, double* lse,
                         const void* q, int q_dtype,
                         const void* k_cache, const void* v_cache, int kv_dtype,
                         const int32_t* block_tables, const int32_t* seq_lens,
                         int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                         int block_size, int max_blocks_per_seq, int num_blocks,
                         double scale, double k_scale, double v_scale,
                         const int32_t* seqs, int n_seqs, int q_len,
                         const float* k_head_scales, const float* v_head_scales);

/* Writes rows `rows` (all num_tokens rows when rows == NULL) of k/v into the caches.
 * FP8 caches: per-tensor k_scale / v_scale, or one scale per KV head when
 * k_head_scales / v_head_scales ([num_kv_heads]) are given (the same in attention). */
int orc_reshape_and_cache(const void* k, const void* v, int in_dtype,
                          void* k_cache, void* v_cache, int kv_dtype,
                          const int64_t* slot_mapping, const int64_t* rows, int64_t n_rows,
                          int num_tokens, int num_kv_heads, int head_dim,
                          int block_size, int num_blocks, float k_scale, float v_scale,
                          const float* k_head_scales, const float* v_head_scales);
#endif
