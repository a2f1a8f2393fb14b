/*
 * ep_oracle.h -- interface of the plain CPU oracle of the EntroPack codec.
 *
 * TEST INFRASTRUCTURE: used only by the tests, the smoke check and the
 * benchmark's CPU-baseline leg.  Private to oracle/; the library has its own,
 * unrelated header.  See ep_oracle.c for the citations and the parity status
 * of every function (which are pinned, which are "parity unpinned").
 */
#ifndef EP_ORACLE_H
#define EP_ORACLE_H
#include <stdint.h>

typedef struct epo_blob epo_blob;

typedef struct {
    double target_bpp;
    int prob_bits;          /* 0: 11 for targets <= 7 bpp, else 12 (App. C.1) */
    int tile_vectors;       /* 0: max(32, floor(S/9)) with S from the target */
    int64_t sample_vectors; /* 0: 2^18 */
    int search_steps;       /* 0: 12 */
    uint64_t seed;          /* 0: shape-dependent seed */
    int has_container_scales;
    int direct_z8;          /* App. A.3 ablation: store z8 instead of m */
    int pooled;             /* App. A.3 ablation: 9 tables, no coset conditioning */
    int rdo_candidates;     /* App. C.2 per-row refinement: K candidate scales (0 or 1: off) */
    int rdo_sweeps;         /* allocation sweeps (0: 1) */
} epo_opts;

void epo_splitmix64(uint64_t seed, int64_t n, uint64_t* out);
void epo_rdo_ratios(int K, double* rho);
uint64_t epo_shape_seed(int64_t rows, int64_t cols);
int64_t epo_sample_rows(int64_t rows, int64_t cols, int64_t sample_vectors, uint64_t seed, int64_t* out_rows);
double epo_row_norm(const float* w, int64_t cols);
int epo_quantize_e8(const double u[8], double y[8]);
void epo_quantize_e8_batch(const double* u, int64_t n, double* y, int32_t* c);
void epo_fields_from_point(const double y[8], int c, int direct_z8, int64_t f[9]);
void epo_point_from_fields(const int64_t f[9], int direct_z8, int64_t y2[8]);
void epo_fields_batch(const double* y, const int32_t* c, int64_t n, int direct_z8, int32_t* fields);
void epo_points_batch(const int32_t* fields, int64_t n, int direct_z8, int32_t* y2);
void epo_normalize_freqs(const uint64_t* count, uint32_t A, uint64_t total, uint32_t M, uint32_t* f);
int64_t epo_default_tile_symbols(double target_bpp);
int64_t epo_tile_vectors(int64_t S);
int64_t epo_tile_metadata_bytes(int64_t ntiles);
float epo_refit_row(const float* w, const double* y, int64_t cols);

int epo_encode(const float* W, int64_t rows, int64_t cols, const epo_opts* opts, epo_blob** out);
int epo_encode_fields(const int32_t* fields, int64_t rows, int64_t cols, const float* row_scales, int b, int V,
                      int flags, epo_blob** out);
double epo_estimate_rate(const float* W, int64_t rows, int64_t cols, const epo_opts* opts, double s, int b);
void epo_free(epo_blob* bl);
void epo_blob_info(const epo_blob* bl, int64_t* ints, double* dbls);
void epo_blob_copy(const epo_blob* bl, uint16_t* payload, uint32_t* tile_index, uint8_t* freq_tables,
                   float* row_scales, int32_t* fields);

uint16_t epo_f32_to_bf16(float x);
uint16_t epo_f32_to_fp16(float x);
uint8_t epo_f32_to_e4m3(float x);
int8_t epo_f32_to_int8(float x);
uint8_t epo_f32_to_uint8(float x);
void epo_convert(const float* in, int64_t n, int dtype, void* out);

int epo_decode_fields(const uint16_t* payload, const uint32_t* tile_index, const uint8_t* freq_tables,
                      int64_t rows, int64_t cols, int64_t t0, int64_t t1, int32_t* fields_out);
int epo_decode(const uint16_t* payload, const uint32_t* tile_index, const uint8_t* freq_tables,
               const float* row_scales, int64_t rows, int64_t cols, int dtype, int64_t t0, int64_t t1, void* out);

#endif
