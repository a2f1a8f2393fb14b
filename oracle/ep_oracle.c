/*
 * ep_oracle.c -- plain CPU oracle of the EntroPack codec.
 *
 * TEST INFRASTRUCTURE.  This file is the independent reference against which the
 * GPU decoder and the CPU packer of the library are checked.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or constant generator with the library, and the library never
 * calls it.
 *
 * Sources ("EntroPack: Fast and Accurate Entropy-Coded Weight Compression at
 * Arbitrary Bitrates", the paper page, cited by section / table):
 *   §1 Introduction            pipeline: row normalisation, E8 blocks of eight,
 *                              invertible integer fields, coset-conditioned model
 *   §3.1 Objective and pipeline encode / decode order
 *   §3.4 Geometric search      bracket update on [lo, hi], geometric midpoint
 *   §3.5 Row-scale refit       one FP32 reconstruction scale per row
 *   §3.6 Frequency tables and tiles, Stored representation
 *   App. A.3                   field tuple (c, z1..z7, m), seventeen tables,
 *                              ablations (pooled tables, direct z8)
 *   App. C.1                   search constants, precision escalation, coarsening
 *   App. C.3                   tile layout, state normalisation, decoder LUTs
 *   Table 5                    tile sizes S -> V and tile metadata bytes
 *   Conway & Sloane (1982)     nearest point of D_n and of E8 = D8 u (D8 + 1/2)
 *
 * Everything is double precision except where the pages fix FP32 (row scales,
 * the reconstruction multiply).  The places where the pages are silent are taken
 * with the plainest reading; each is marked READING below.
 *
 * Parity status of each function:
 *   pinned    quantize_e8 (brute force, covering radius, Q(y)=y), fields
 *             (exhaustive bijection), rANS coder (round trip, terminal states,
 *             cursor, code length near the entropy), tile layout (Table 5),
 *             dtype conversions (library conversions; the INT8 and UINT8
 *             readings on their own edge cases and numpy), splitmix64 (published
 *             outputs), refit (least-squares optimality), normalize_freqs
 *             (hand-worked counts -> frequencies of the reading below; sum,
 *             support and coding-loss invariants on random counts),
 *             sample_rows (a partial Fisher-Yates draw worked by hand from
 *             published generator outputs; draws uniform over orders and rows),
 *             scale search (rate lands near target, bracket property), stored
 *             bytes (closed form).
 *   parity unpinned (readings with no page value to check against; the pins
 *             above check that the code follows each reading, not the reading
 *             itself): the choice
 *             of row normaliser (RMS), the frequency normalisation rule, the
 *             sampling generator and order, the tie-breaks, the lane interleave
 *             order and the header byte layout.  They change the encoder's
 *             choices, never the decoder's arithmetic on a given stream.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "ep_oracle.h"

#define J_LANES 32               /* App. C.3: J = 32 interleaved states per tile */
#define STATE_LOW (1u << 15)     /* App. C.3: states kept in [2^15, 2^31)        */
#define NFIELDS 9                /* App. A.3: (c, z1..z7, m)                    */
#define MAX_TABLES 17            /* App. A.3: 1 + 2 x 8                          */
#define HDR_FIXED 48
#define MAGIC 0x314B5045u        /* "EPK1" */

/* ------------------------------------------------------------------------ */
/* small helpers                                                            */
/* ------------------------------------------------------------------------ */

static void put_u32(uint8_t* p, uint32_t v) {
    p[0] = (uint8_t)(v & 0xFF);
    p[1] = (uint8_t)((v >> 8) & 0xFF);
    p[2] = (uint8_t)((v >> 16) & 0xFF);
    p[3] = (uint8_t)((v >> 24) & 0xFF);
}
static void put_u64(uint8_t* p, uint64_t v) {
    put_u32(p, (uint32_t)(v & 0xFFFFFFFFu));
    put_u32(p + 4, (uint32_t)(v >> 32));
}
static uint32_t get_u32(const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t get_u64(const uint8_t* p) {
    return (uint64_t)get_u32(p) | ((uint64_t)get_u32(p + 4) << 32);
}
static uint16_t get_u16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* ------------------------------------------------------------------------ */
/* splitmix64 (Steele, Lea & Flood 2014; Vigna's public-domain reference).  */
/* Drives the sampled-row selection of App. C.1 ("shape-dependent seed").   */
/* ------------------------------------------------------------------------ */

static uint64_t splitmix64_next(uint64_t* state) {
    uint64_t z;
    *state += 0x9E3779B97F4A7C15ull;
    z = *state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

void epo_splitmix64(uint64_t seed, int64_t n, uint64_t* out) {
    uint64_t st = seed;
    for (int64_t i = 0; i < n; ++i) out[i] = splitmix64_next(&st);
}

/* READING: without a user seed, the shape-dependent seed is rows * 2^32 xor cols. */
uint64_t epo_shape_seed(int64_t rows, int64_t cols) {
    return ((uint64_t)rows << 32) ^ (uint64_t)cols;
}

/*
 * Sampled rate evaluation (App. C.1): complete rows, nominal budget of
 * sample_vectors eight-dimensional vectors, fixed for the whole search.
 * READING: Rs = min(rows, ceil(sample_vectors / ceil(cols/8))) rows drawn without
 * replacement by a partial Fisher-Yates shuffle; r_i = i + (next mod (rows - i)).
 * Returns Rs; out_rows receives the chosen rows in draw order.
 */
int64_t epo_sample_rows(int64_t rows, int64_t cols, int64_t sample_vectors, uint64_t seed,
                        int64_t* out_rows) {
    int64_t nq = ceil_div(cols, 8);
    int64_t rs = ceil_div(sample_vectors, nq);
    if (rs > rows) rs = rows;
    if (rs < 1) rs = 1;
    int64_t* perm = (int64_t*)malloc(sizeof(int64_t) * (size_t)rows);
    for (int64_t i = 0; i < rows; ++i) perm[i] = i;
    uint64_t st = seed ? seed : epo_shape_seed(rows, cols);
    for (int64_t i = 0; i < rs; ++i) {
        uint64_t r = splitmix64_next(&st);
        int64_t j = i + (int64_t)(r % (uint64_t)(rows - i));
        int64_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
        out_rows[i] = perm[i];
    }
    free(perm);
    return rs;
}

/* ------------------------------------------------------------------------ */
/* A1  Row normalisation (§1, §3.2 heading).                                */
/* READING: the normaliser is the row RMS, sqrt(mean_j w_j^2), summed in     */
/* index order in double; an all-zero row uses 1.                           */
/* ------------------------------------------------------------------------ */

double epo_row_norm(const float* w, int64_t cols) {
    double acc = 0.0;
    for (int64_t j = 0; j < cols; ++j) acc += (double)w[j] * (double)w[j];
    double n = sqrt(acc / (double)cols);
    return n > 0.0 ? n : 1.0;
}

/* ------------------------------------------------------------------------ */
/* A2  Nearest point of E8 (Conway & Sloane 1982).                          */
/* ------------------------------------------------------------------------ */

/*
 * Nearest point of D8 = {a in Z^8 : sum a even}: round every coordinate to the
 * nearest integer (ties to even); if the sum is odd, round the coordinate that
 * was furthest from an integer the other way.  READING (tie-breaks): the lowest
 * index wins among equally far coordinates; a coordinate with u - a >= 0 moves
 * up, otherwise down.  Any of these choices gives a nearest point.
 */
static void nearest_d8(const double u[8], double a[8]) {
    long long sum = 0;
    for (int k = 0; k < 8; ++k) {
        a[k] = nearbyint(u[k]); /* default rounding mode: to nearest, ties to even */
        sum += (long long)a[k];
    }
    if (sum & 1LL) {
        int kbest = 0;
        double dbest = -1.0;
        for (int k = 0; k < 8; ++k) {
            double d = fabs(u[k] - a[k]);
            if (d > dbest) {
                dbest = d;
                kbest = k;
            }
        }
        a[kbest] += (u[kbest] - a[kbest] >= 0.0) ? 1.0 : -1.0;
    }
}

/*
 * E8 = D8 u (D8 + 1/2): decode u in both cosets and keep the nearer point
 * (READING: ties go to D8).  Returns the coset bit c (0: D8, 1: D8 + 1/2).
 */
int epo_quantize_e8(const double u[8], double y[8]) {
    double a[8], b[8], v[8];
    nearest_d8(u, a);
    for (int k = 0; k < 8; ++k) v[k] = u[k] - 0.5;
    nearest_d8(v, b);
    for (int k = 0; k < 8; ++k) b[k] += 0.5;
    double da = 0.0, db = 0.0;
    for (int k = 0; k < 8; ++k) {
        da += (u[k] - a[k]) * (u[k] - a[k]);
        db += (u[k] - b[k]) * (u[k] - b[k]);
    }
    if (db < da) {
        memcpy(y, b, sizeof(b));
        return 1;
    }
    memcpy(y, a, sizeof(a));
    return 0;
}

void epo_quantize_e8_batch(const double* u, int64_t n, double* y, int32_t* c) {
    for (int64_t i = 0; i < n; ++i) c[i] = epo_quantize_e8(u + 8 * i, y + 8 * i);
}

/* ------------------------------------------------------------------------ */
/* A3  Invertible integer fields (§1, App. A.3, the parity reduction).       */
/* c: coset bit; z = y - c/2 lies in D8 (integer, even sum) in both cosets;  */
/* p = (z1 + ... + z7) mod 2; m = (z8 - p) / 2 replaces z8.                  */
/* direct_z8 = 1 gives the App. A.3 ablation that stores z8 itself.          */
/* ------------------------------------------------------------------------ */

void epo_fields_from_point(const double y[8], int c, int direct_z8, int64_t f[NFIELDS]) {
    int64_t z[8];
    for (int k = 0; k < 8; ++k) z[k] = (int64_t)(y[k] - 0.5 * (double)c);
    int64_t s7 = 0;
    for (int k = 0; k < 7; ++k) s7 += z[k];
    int64_t p = ((s7 % 2) + 2) % 2;
    f[0] = c;
    for (int k = 0; k < 7; ++k) f[1 + k] = z[k];
    f[8] = direct_z8 ? z[7] : (z[7] - p) / 2;
}

/* Inverse: z8 = 2m + p, y = z + c/2.  Returns 2y (integers) to stay exact. */
void epo_point_from_fields(const int64_t f[NFIELDS], int direct_z8, int64_t y2[8]) {
    int64_t c = f[0];
    int64_t z[8];
    int64_t s7 = 0;
    for (int k = 0; k < 7; ++k) {
        z[k] = f[1 + k];
        s7 += z[k];
    }
    int64_t p = ((s7 % 2) + 2) % 2;
    z[7] = direct_z8 ? f[8] : 2 * f[8] + p;
    for (int k = 0; k < 8; ++k) y2[k] = 2 * z[k] + c;
}

void epo_fields_batch(const double* y, const int32_t* c, int64_t n, int direct_z8, int32_t* fields) {
    int64_t f[NFIELDS];
    for (int64_t i = 0; i < n; ++i) {
        epo_fields_from_point(y + 8 * i, c[i], direct_z8, f);
        for (int k = 0; k < NFIELDS; ++k) fields[NFIELDS * i + k] = (int32_t)f[k];
    }
}

void epo_points_batch(const int32_t* fields, int64_t n, int direct_z8, int32_t* y2) {
    int64_t f[NFIELDS], o[8];
    for (int64_t i = 0; i < n; ++i) {
        for (int k = 0; k < NFIELDS; ++k) f[k] = fields[NFIELDS * i + k];
        epo_point_from_fields(f, direct_z8, o);
        for (int k = 0; k < 8; ++k) y2[8 * i + k] = (int32_t)o[k];
    }
}

/* ------------------------------------------------------------------------ */
/* A4  Coset-conditioned model: which table codes field k (App. A.3).        */
/* 17 tables: table 0 for c; table 1 + 2(k-1) + c for field k = 1..8.        */
/* pooled (the App. A.3 ablation, 9 tables): table k for field k.            */
/* ------------------------------------------------------------------------ */

static int table_of(int field, int c, int pooled) {
    if (field == 0) return 0;
    return pooled ? field : 1 + 2 * (field - 1) + c;
}

/* ------------------------------------------------------------------------ */
/* A11 Frequency tables normalised to M = 2^b (§3.6, App. C.1).              */
/* READING: f = max(1, floor(count*M/total + 1/2)) for observed symbols and  */
/* 0 otherwise; while the sum exceeds M, lower the largest f > 1 by one      */
/* (lowest symbol on ties); while it is short, raise the most frequent       */
/* symbol (lowest symbol on ties).  Requires 1 <= A <= M.                    */
/* ------------------------------------------------------------------------ */

void epo_normalize_freqs(const uint64_t* count, uint32_t A, uint64_t total, uint32_t M, uint32_t* f) {
    uint64_t sum = 0;
    for (uint32_t s = 0; s < A; ++s) {
        if (count[s] == 0) {
            f[s] = 0;
        } else {
            double q = (double)count[s] * (double)M / (double)total;
            double r = floor(q + 0.5);
            f[s] = r < 1.0 ? 1u : (uint32_t)r;
        }
        sum += f[s];
    }
    while (sum > M) {
        uint32_t best = A;
        for (uint32_t s = 0; s < A; ++s)
            if (f[s] > 1 && (best == A || f[s] > f[best])) best = s;
        if (best == A) break; /* cannot happen when A <= M */
        f[best] -= 1;
        sum -= 1;
    }
    while (sum < M) {
        uint32_t best = 0;
        for (uint32_t s = 1; s < A; ++s)
            if (count[s] > count[best]) best = s;
        f[best] += 1;
        sum += 1;
    }
}

/* One table: alphabet [min, min + A), frequencies at precision b. */
typedef struct {
    int32_t min;
    uint32_t A;
    uint64_t total;
    uint64_t* count;
    uint32_t* freq;
    uint32_t* cum;
} table_t;

static void table_free(table_t* t) {
    free(t->count);
    free(t->freq);
    free(t->cum);
    memset(t, 0, sizeof(*t));
}

/*
 * Count the fields of vectors [0, nvec) into ntab tables.  Field values are
 * taken from fields[9*g + k].  Returns the largest coordinate alphabet.
 * When the largest alphabet exceeds amax_limit the counts are not built
 * (the caller only needs to know that the alphabet does not fit).
 */
static uint64_t count_tables(const int32_t* fields, int64_t nvec, int pooled, int ntab,
                             uint64_t amax_limit, table_t* tabs) {
    int64_t lo[MAX_TABLES], hi[MAX_TABLES];
    for (int t = 0; t < ntab; ++t) {
        lo[t] = INT64_MAX;
        hi[t] = INT64_MIN;
    }
    for (int64_t g = 0; g < nvec; ++g) {
        const int32_t* f = fields + NFIELDS * g;
        for (int k = 0; k < NFIELDS; ++k) {
            int t = table_of(k, f[0], pooled);
            if (f[k] < lo[t]) lo[t] = f[k];
            if (f[k] > hi[t]) hi[t] = f[k];
        }
    }
    uint64_t amax = 0;
    for (int t = 1; t < ntab; ++t)
        if (hi[t] >= lo[t] && (uint64_t)(hi[t] - lo[t] + 1) > amax) amax = (uint64_t)(hi[t] - lo[t] + 1);
    for (int t = 0; t < ntab; ++t) {
        memset(&tabs[t], 0, sizeof(table_t));
        if (hi[t] < lo[t]) continue; /* empty table: A = 0 */
        tabs[t].min = (int32_t)lo[t];
        tabs[t].A = (uint32_t)(hi[t] - lo[t] + 1);
    }
    if (amax > amax_limit) return amax;
    for (int t = 0; t < ntab; ++t) tabs[t].count = (uint64_t*)calloc(tabs[t].A ? tabs[t].A : 1, sizeof(uint64_t));
    for (int64_t g = 0; g < nvec; ++g) {
        const int32_t* f = fields + NFIELDS * g;
        for (int k = 0; k < NFIELDS; ++k) {
            int t = table_of(k, f[0], pooled);
            tabs[t].count[f[k] - tabs[t].min] += 1;
            tabs[t].total += 1;
        }
    }
    return amax;
}

static void build_freqs(table_t* tabs, int ntab, int b) {
    uint32_t M = 1u << b;
    for (int t = 0; t < ntab; ++t) {
        table_t* tb = &tabs[t];
        tb->freq = (uint32_t*)calloc(tb->A ? tb->A : 1, sizeof(uint32_t));
        tb->cum = (uint32_t*)calloc((tb->A ? tb->A : 1) + 1, sizeof(uint32_t));
        if (tb->A == 0) continue;
        epo_normalize_freqs(tb->count, tb->A, tb->total, M, tb->freq);
        tb->cum[0] = 0;
        for (uint32_t s = 0; s < tb->A; ++s) tb->cum[s + 1] = tb->cum[s] + tb->freq[s];
    }
}

/* ------------------------------------------------------------------------ */
/* A13 Tile sizing (App. C.3, Table 5): V = max(32, floor(S/9)).             */
/* READING: S by target rate, fitted to Table 5's four rows:                 */
/* 32768 up to 2.5 bpp, 16384 up to 5, 8192 up to 7, 4096 above.            */
/* ------------------------------------------------------------------------ */

int64_t epo_default_tile_symbols(double target_bpp) {
    if (target_bpp <= 2.5) return 32768;
    if (target_bpp <= 5.0) return 16384;
    if (target_bpp <= 7.0) return 8192;
    return 4096;
}

int64_t epo_tile_vectors(int64_t S) {
    int64_t v = S / 9;
    return v > 32 ? v : 32;
}

/* Tile metadata bytes (App. C.3): T * (4J + 4) + one final boundary offset. */
int64_t epo_tile_metadata_bytes(int64_t ntiles) { return ntiles * (4 * J_LANES + 4) + 4; }

static int64_t header_bytes(int ntab) {
    int64_t h = HDR_FIXED + 8 * (int64_t)ntab;
    return (h + 15) / 16 * 16;
}

/* ------------------------------------------------------------------------ */
/* Quantisation of whole rows at scale s: u = (w / n_r) / s, y = Q_E8(u).   */
/* READING (cols % 8 != 0): the row is padded with zeros to whole vectors;  */
/* the padding is quantised with its vector and dropped by the decoder.     */
/* ------------------------------------------------------------------------ */

static void quantize_row(const float* w, int64_t cols, double norm, double s, int direct_z8,
                         int32_t* fields_out, double* y_out /* nullable, 8 per vector */) {
    double u[8], y[8];
    int64_t f[NFIELDS];
    for (int64_t q = 0; q < ceil_div(cols, 8); ++q) {
        for (int k = 0; k < 8; ++k) u[k] = 8 * q + k < cols ? ((double)w[8 * q + k] / norm) / s : 0.0;
        int c = epo_quantize_e8(u, y);
        epo_fields_from_point(y, c, direct_z8, f);
        for (int k = 0; k < NFIELDS; ++k) fields_out[NFIELDS * q + k] = (int32_t)f[k];
        if (y_out) memcpy(y_out + 8 * q, y, sizeof(y));
    }
}

/* ------------------------------------------------------------------------ */
/* A5/A6 Stored-size estimate from the sampled rows (§3.4, App. C.1).        */
/* READING: payload bits = (nvec / nvec_sample) * sum over the sample's      */
/* symbols of -log2(f/M) under tables built from the sample; side bytes are  */
/* exact (header, tables, tile metadata, row scales, container scales).      */
/* An alphabet wider than 2^b makes the estimate +inf.                       */
/* ------------------------------------------------------------------------ */

typedef struct {
    int64_t rows, cols, nvec, ntiles;
    int pooled, direct_z8, ntab;
    int has_container_scales;
} shape_t;

static int64_t side_bytes(const shape_t* sh, const table_t* tabs) {
    int64_t tb = header_bytes(sh->ntab);
    for (int t = 0; t < sh->ntab; ++t) tb += 2 * (int64_t)tabs[t].A;
    int64_t side = tb + epo_tile_metadata_bytes(sh->ntiles) + 4 * sh->rows;
    if (sh->has_container_scales) side += 4 * sh->rows;
    return side;
}

static double estimate_rate(const shape_t* sh, const float* W, const double* norms,
                            const int64_t* srows, int64_t rs, double s, int b, int32_t* scratch_fields) {
    int64_t nq = ceil_div(sh->cols, 8);
    for (int64_t i = 0; i < rs; ++i) {
        int64_t r = srows[i];
        quantize_row(W + r * sh->cols, sh->cols, norms[r], s, sh->direct_z8, scratch_fields + NFIELDS * nq * i, NULL);
    }
    int64_t nsamp = rs * nq;
    table_t tabs[MAX_TABLES];
    uint64_t amax = count_tables(scratch_fields, nsamp, sh->pooled, sh->ntab, 1u << b, tabs);
    double rate;
    if (amax > (1u << b)) {
        rate = INFINITY;
    } else {
        build_freqs(tabs, sh->ntab, b);
        double bits = 0.0;
        for (int t = 0; t < sh->ntab; ++t)
            for (uint32_t k = 0; k < tabs[t].A; ++k)
                if (tabs[t].count[k]) bits += (double)tabs[t].count[k] * ((double)b - log2((double)tabs[t].freq[k]));
        double payload_bytes = bits / 8.0 * ((double)sh->nvec / (double)nsamp);
        double total = payload_bytes + (double)side_bytes(sh, tabs);
        rate = 8.0 * total / (double)(sh->rows * sh->cols); /* per real weight */
    }
    for (int t = 0; t < sh->ntab; ++t) table_free(&tabs[t]);
    return rate;
}

/* ------------------------------------------------------------------------ */
/* Interleaved rANS over one tile (§3.6, App. C.3).                          */
/* READING (interleave): vector v of a tile belongs to lane v mod 32; decode */
/* step t = 9r + f decodes field f of vector 32r + j on every lane j with    */
/* 32r + j < V_t; within a step, lanes that renormalise read consecutive     */
/* payload words in ascending lane order.                                    */
/* State x in [2^15, 2^31), 16-bit words, M = 2^b <= 2^15.                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    uint16_t* w;
    int64_t n, cap;
} wordbuf_t;

static void wb_push(wordbuf_t* b, uint16_t v) {
    if (b->n == b->cap) {
        b->cap = b->cap ? 2 * b->cap : 1024;
        b->w = (uint16_t*)realloc(b->w, sizeof(uint16_t) * (size_t)b->cap);
    }
    b->w[b->n++] = v;
}

/* Encode tile [v0, v0 + vt); appends the tile's payload words to out and writes 32 states. */
static void rans_encode_tile(const int32_t* fields, int64_t v0, int64_t vt, const table_t* tabs, int b, int pooled,
                             wordbuf_t* out, uint32_t states[J_LANES]) {
    uint64_t x[J_LANES];
    uint32_t M = 1u << b;
    wordbuf_t em = {0, 0, 0};
    for (int j = 0; j < J_LANES; ++j) x[j] = STATE_LOW;
    int64_t rounds = ceil_div(vt, J_LANES);
    for (int64_t step = NFIELDS * rounds - 1; step >= 0; --step) {
        int64_t r = step / NFIELDS;
        int fld = (int)(step % NFIELDS);
        for (int j = J_LANES - 1; j >= 0; --j) {
            int64_t v = J_LANES * r + j;
            if (v >= vt) continue;
            const int32_t* f = fields + NFIELDS * (v0 + v);
            const table_t* tb = &tabs[table_of(fld, f[0], pooled)];
            uint32_t sym = (uint32_t)(f[fld] - tb->min);
            uint64_t fr = tb->freq[sym], cm = tb->cum[sym];
            uint64_t xmax = fr << (31 - b);
            if (x[j] >= xmax) {
                wb_push(&em, (uint16_t)(x[j] & 0xFFFF));
                x[j] >>= 16;
            }
            x[j] = (x[j] / fr) * M + (x[j] % fr) + cm;
        }
    }
    for (int64_t i = em.n - 1; i >= 0; --i) wb_push(out, em.w[i]);
    for (int j = 0; j < J_LANES; ++j) states[j] = (uint32_t)x[j];
    free(em.w);
}

/* ------------------------------------------------------------------------ */
/* The stored blob.                                                          */
/* ------------------------------------------------------------------------ */

struct epo_blob {
    int64_t rows, cols, nvec;
    int b, V, ntiles, ntab, flags;
    double s, stored_bpp, target_bpp;
    int64_t stored_bytes;
    uint16_t* payload;
    int64_t payload_words;
    uint32_t* tile_index; /* 33 * ntiles + 1 */
    uint8_t* freq_tables;
    int64_t freq_bytes;
    float* row_scales;
    int32_t* fields; /* 9 * nvec, the encoder's fields (for tests) */
    int has_container_scales;
};

void epo_free(epo_blob* bl) {
    if (!bl) return;
    free(bl->payload);
    free(bl->tile_index);
    free(bl->freq_tables);
    free(bl->row_scales);
    free(bl->fields);
    free(bl);
}

/* Serialise the tables: fixed header, ntab x {i32 min, u32 A}, u16 frequencies. */
static void write_tables(epo_blob* bl, const table_t* tabs) {
    int64_t hb = header_bytes(bl->ntab);
    int64_t nf = 0;
    for (int t = 0; t < bl->ntab; ++t) nf += tabs[t].A;
    bl->freq_bytes = hb + 2 * nf;
    bl->freq_tables = (uint8_t*)calloc((size_t)bl->freq_bytes, 1);
    uint8_t* p = bl->freq_tables;
    put_u32(p + 0, MAGIC);
    put_u32(p + 4, 1);
    put_u32(p + 8, (uint32_t)bl->b);
    put_u32(p + 12, (uint32_t)bl->V);
    put_u32(p + 16, J_LANES);
    put_u32(p + 20, (uint32_t)bl->ntiles);
    put_u64(p + 24, (uint64_t)bl->rows);
    put_u64(p + 32, (uint64_t)bl->cols);
    put_u32(p + 40, (uint32_t)bl->ntab);
    put_u32(p + 44, (uint32_t)bl->flags);
    for (int t = 0; t < bl->ntab; ++t) {
        put_u32(p + HDR_FIXED + 8 * t, (uint32_t)tabs[t].min);
        put_u32(p + HDR_FIXED + 8 * t + 4, tabs[t].A);
    }
    int64_t o = hb;
    for (int t = 0; t < bl->ntab; ++t)
        for (uint32_t s = 0; s < tabs[t].A; ++s) {
            uint32_t v = tabs[t].freq[s];
            p[o] = (uint8_t)(v & 0xFF);
            p[o + 1] = (uint8_t)(v >> 8);
            o += 2;
        }
}

/*
 * Entropy-code given fields (rows x ceil(cols/8) vectors, 9 fields each) with given
 * row scales: tables from the counts over the whole tensor's final fields
 * (§3.6), tiles of V vectors, interleaved rANS per tile.
 * Returns 0, or a negative code when an alphabet exceeds 2^b.
 */
static int code_fields(epo_blob* bl, int pooled) {
    table_t tabs[MAX_TABLES];
    uint64_t amax = count_tables(bl->fields, bl->nvec, pooled, bl->ntab, 1u << bl->b, tabs);
    if (amax > (1u << bl->b)) {
        for (int t = 0; t < bl->ntab; ++t) table_free(&tabs[t]);
        return -3;
    }
    build_freqs(tabs, bl->ntab, bl->b);
    bl->ntiles = (int)ceil_div(bl->nvec, bl->V);
    bl->tile_index = (uint32_t*)calloc((size_t)(33 * (int64_t)bl->ntiles + 1), sizeof(uint32_t));
    wordbuf_t pay = {0, 0, 0};
    for (int64_t t = 0; t < bl->ntiles; ++t) {
        int64_t v0 = t * bl->V;
        int64_t vt = bl->nvec - v0 < bl->V ? bl->nvec - v0 : bl->V;
        bl->tile_index[33 * t] = (uint32_t)pay.n;
        rans_encode_tile(bl->fields, v0, vt, tabs, bl->b, pooled, &pay, bl->tile_index + 33 * t + 1);
    }
    bl->tile_index[33 * (int64_t)bl->ntiles] = (uint32_t)pay.n;
    bl->payload = pay.w ? pay.w : (uint16_t*)calloc(1, sizeof(uint16_t));
    bl->payload_words = pay.n;
    write_tables(bl, tabs);
    for (int t = 0; t < bl->ntab; ++t) table_free(&tabs[t]);
    bl->stored_bytes = 2 * bl->payload_words + 4 * (33 * (int64_t)bl->ntiles + 1) + bl->freq_bytes + 4 * bl->rows +
                       (bl->has_container_scales ? 4 * bl->rows : 0);
    bl->stored_bpp = 8.0 * (double)bl->stored_bytes / (double)(bl->rows * bl->cols);
    return 0;
}

/*
 * Code caller-given fields (tests of the coder alone).  fields: 9 per vector.
 * b in [9, 15], V >= 1.  flags bit0 = direct z8, bit1 = pooled tables.
 */
int epo_encode_fields(const int32_t* fields, int64_t rows, int64_t cols, const float* row_scales, int b, int V,
                      int flags, epo_blob** out) {
    *out = NULL;
    if (rows <= 0 || cols <= 0 || b < 9 || b > 15 || V < 1) return -1;
    epo_blob* bl = (epo_blob*)calloc(1, sizeof(epo_blob));
    bl->rows = rows;
    bl->cols = cols;
    bl->nvec = rows * ceil_div(cols, 8);
    bl->b = b;
    bl->V = V;
    bl->flags = flags;
    bl->ntab = (flags & 2) ? 9 : 17;
    bl->fields = (int32_t*)malloc(sizeof(int32_t) * (size_t)(NFIELDS * bl->nvec));
    memcpy(bl->fields, fields, sizeof(int32_t) * (size_t)(NFIELDS * bl->nvec));
    bl->row_scales = (float*)malloc(sizeof(float) * (size_t)rows);
    memcpy(bl->row_scales, row_scales, sizeof(float) * (size_t)rows);
    int rc = code_fields(bl, (flags & 2) != 0);
    if (rc) {
        epo_free(bl);
        return rc;
    }
    *out = bl;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Full encoder (§3.1 pipeline; Algorithm 1 as described in §3.4 / C.1).     */
/* ------------------------------------------------------------------------ */

/*
 * A9 Row-scale refit (§3.5 heading, §3.1 "fit one reconstruction scale per row").
 * READING: least squares in the original weight units, sigma_r =
 * fl32(<w_r, y_r> / <y_r, y_r>) with sums in index order in double; 0 when y_r = 0.
 */
float epo_refit_row(const float* w, const double* y, int64_t cols) {
    double num = 0.0, den = 0.0;
    for (int64_t j = 0; j < cols; ++j) {
        num += (double)w[j] * y[j];
        den += y[j] * y[j];
    }
    if (den == 0.0) return 0.0f;
    return (float)(num / den);
}

/*
 * A10 Per-row rate-distortion refinement ([paper] §3.5: each row picks one of
 * several quantisation steps, all rows sharing one storage budget; App. C.2;
 * Figs. 3-4).  Off unless asked for ([paper] §4.1 runs it in its own ablations
 * only).
 *
 * Candidate ratios (§3.5): K ratios in [0.70, 1.45], starting from 1; each
 * further ratio bisects, in log scale, the widest interval between neighbouring
 * ratios and the ends of the range.  READING: the ends are not candidates
 * themselves; ties between equally wide intervals go to the lower interval.
 */
void epo_rdo_ratios(int K, double* rho) {
    double pts[2 + 64];
    int n = 3;
    pts[0] = 0.70;
    pts[1] = 1.0;
    pts[2] = 1.45;
    rho[0] = 1.0;
    for (int k = 1; k < K && k < 64; ++k) {
        int best = 0;
        double wbest = -1.0;
        for (int i = 0; i + 1 < n; ++i) {
            double w = log(pts[i + 1] / pts[i]);
            if (w > wbest) {
                wbest = w;
                best = i;
            }
        }
        double mid = sqrt(pts[best] * pts[best + 1]);
        for (int i = n; i > best + 1; --i) pts[i] = pts[i - 1];
        pts[best + 1] = mid;
        ++n;
        rho[k] = mid;
    }
}

/* Ideal code length of one row's fields under the tables: sum over its symbols, in
 * order, of b - log2 f, with f = 1 for a symbol the table gives no frequency
 * (READING: an unseen symbol costs the minimum frequency, b bits). */
static double row_bits(const int32_t* f, int64_t nq, const table_t* tabs, int b, int pooled) {
    double bits = 0.0;
    for (int64_t q = 0; q < nq; ++q) {
        const int32_t* v = f + NFIELDS * q;
        for (int k = 0; k < NFIELDS; ++k) {
            const table_t* tb = &tabs[table_of(k, v[0], pooled)];
            int64_t i = (int64_t)v[k] - tb->min;
            uint32_t fr = (tb->A && i >= 0 && i < (int64_t)tb->A) ? tb->freq[i] : 0u;
            bits += (double)b - log2((double)(fr ? fr : 1u));
        }
    }
    return bits;
}

/*
 * App. C.2 allocation.  READINGS: candidate k of row r quantises the row at
 * rho_k s (the row normaliser unchanged) and refits its scale (A9); its
 * distortion is sum_j (w_j - sigma y_j)^2 in weight units (sigma as stored, FP32).
 * A candidate is admissible when every symbol lies in the baseline tables'
 * alphabets (so the stored alphabets keep fitting 2^b).  Budget: the baseline's
 * ideal code length under its own tables.  A sweep prices every admissible
 * candidate under the current tables, finds the smallest common rate penalty
 * lambda (64 bisection steps of log2 lambda on [-80, 80]) whose per-row choices
 * argmin D + lambda R (ties: lowest k) fit the budget, and rebuilds the tables
 * from the chosen fields.  In: fields at ratio 1; out: chosen fields and scales.
 */
static void rdo_refine(const shape_t* sh, const float* W, const double* norms, double s, int b, int K, int sweeps,
                       int32_t* fields, float* scales) {
    const int64_t rows = sh->rows, cols = sh->cols, nq = ceil_div(cols, 8), rowf = NFIELDS * nq;
    double rho[64];
    if (K > 64) K = 64;
    epo_rdo_ratios(K, rho);
    int32_t* cf = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K * rows * rowf));
    float* cs = (float*)malloc(sizeof(float) * (size_t)(K * rows));
    double* cd = (double*)malloc(sizeof(double) * (size_t)(K * rows));
    double* cr = (double*)malloc(sizeof(double) * (size_t)(K * rows));
    unsigned char* ok = (unsigned char*)malloc((size_t)(K * rows));
    int* sel = (int*)malloc(sizeof(int) * (size_t)rows);
    double* y = (double*)malloc(sizeof(double) * (size_t)(8 * nq));
    table_t base[MAX_TABLES], tabs[MAX_TABLES];
    count_tables(fields, sh->nvec, sh->pooled, sh->ntab, UINT64_MAX, base);
    build_freqs(base, sh->ntab, b);
    for (int k = 0; k < K; ++k)
        for (int64_t r = 0; r < rows; ++r) {
            const float* w = W + r * cols;
            int32_t* f = cf + (k * rows + r) * rowf;
            quantize_row(w, cols, norms[r], rho[k] * s, sh->direct_z8, f, y);
            float sg = epo_refit_row(w, y, cols);
            double d = 0.0;
            for (int64_t j = 0; j < cols; ++j) {
                double e = (double)w[j] - (double)sg * y[j];
                d += e * e;
            }
            cs[k * rows + r] = sg;
            cd[k * rows + r] = d;
            unsigned char in = 1;
            for (int64_t q = 0; q < nq && in; ++q)
                for (int m = 0; m < NFIELDS; ++m) {
                    const table_t* tb = &base[table_of(m, f[NFIELDS * q], sh->pooled)];
                    int64_t i = (int64_t)f[NFIELDS * q + m] - tb->min;
                    if (!tb->A || i < 0 || i >= (int64_t)tb->A) in = 0;
                }
            ok[k * rows + r] = in;
        }
    double budget = 0.0;
    for (int64_t r = 0; r < rows; ++r) budget += row_bits(cf + r * rowf, nq, base, b, sh->pooled);
    for (int64_t r = 0; r < rows; ++r) sel[r] = 0;
    const table_t* model = base;
    for (int sw = 0; sw < sweeps; ++sw) {
        for (int k = 0; k < K; ++k)
            for (int64_t r = 0; r < rows; ++r)
                cr[k * rows + r] = ok[k * rows + r] ? row_bits(cf + (k * rows + r) * rowf, nq, model, b, sh->pooled)
                                                    : INFINITY;
        double lo = -80.0, hi = 80.0;
        for (int it = 0; it <= 64; ++it) {
            double t = it < 64 ? 0.5 * (lo + hi) : hi; /* the last pass applies the final lambda */
            double lam = exp2(t), total = 0.0;
            for (int64_t r = 0; r < rows; ++r) {
                int best = 0;
                double jbest = cd[r] + lam * cr[r];
                for (int k = 1; k < K; ++k) {
                    double j = cd[k * rows + r] + lam * cr[k * rows + r];
                    if (j < jbest) {
                        jbest = j;
                        best = k;
                    }
                }
                sel[r] = best;
                total += cr[best * rows + r];
            }
            if (it < 64) {
                if (total <= budget) hi = t;
                else lo = t;
            }
        }
        for (int64_t r = 0; r < rows; ++r)
            memcpy(fields + r * rowf, cf + (sel[r] * rows + r) * rowf, sizeof(int32_t) * (size_t)rowf);
        if (model != base)
            for (int t = 0; t < sh->ntab; ++t) table_free(&tabs[t]);
        count_tables(fields, sh->nvec, sh->pooled, sh->ntab, UINT64_MAX, tabs);
        build_freqs(tabs, sh->ntab, b);
        model = tabs;
    }
    for (int64_t r = 0; r < rows; ++r) scales[r] = cs[sel[r] * rows + r];
    for (int t = 0; t < sh->ntab; ++t) table_free(&base[t]);
    if (model != base)
        for (int t = 0; t < sh->ntab; ++t) table_free(&tabs[t]);
    free(cf); free(cs); free(cd); free(cr); free(ok); free(sel); free(y);
}

int epo_encode(const float* W, int64_t rows, int64_t cols, const epo_opts* opts, epo_blob** out) {
    *out = NULL;
    if (rows <= 0 || cols <= 0) return -1;
    if (!(opts->target_bpp > 0.0)) return -1;
    int flags = (opts->direct_z8 ? 1 : 0) | (opts->pooled ? 2 : 0);
    shape_t sh;
    sh.rows = rows;
    sh.cols = cols;
    sh.nvec = rows * ceil_div(cols, 8);
    sh.pooled = opts->pooled != 0;
    sh.direct_z8 = opts->direct_z8 != 0;
    sh.ntab = sh.pooled ? 9 : 17;
    sh.has_container_scales = opts->has_container_scales != 0;
    int64_t V = opts->tile_vectors > 0 ? opts->tile_vectors : epo_tile_vectors(epo_default_tile_symbols(opts->target_bpp));
    sh.ntiles = ceil_div(sh.nvec, V);
    int64_t nq = ceil_div(cols, 8);

    double* norms = (double*)malloc(sizeof(double) * (size_t)rows);
    for (int64_t r = 0; r < rows; ++r) norms[r] = epo_row_norm(W + r * cols, cols);

    int64_t sv = opts->sample_vectors > 0 ? opts->sample_vectors : (1 << 18);
    int64_t* srows = (int64_t*)malloc(sizeof(int64_t) * (size_t)rows);
    int64_t rs = epo_sample_rows(rows, cols, sv, opts->seed, srows);
    int32_t* sfields = (int32_t*)malloc(sizeof(int32_t) * (size_t)(NFIELDS * nq * rs));

    epo_blob* bl = (epo_blob*)calloc(1, sizeof(epo_blob));
    bl->rows = rows;
    bl->cols = cols;
    bl->nvec = sh.nvec;
    bl->V = (int)V;
    bl->flags = flags;
    bl->ntab = sh.ntab;
    bl->target_bpp = opts->target_bpp;
    bl->has_container_scales = sh.has_container_scales;
    bl->fields = (int32_t*)malloc(sizeof(int32_t) * (size_t)(NFIELDS * sh.nvec));
    double* ys = (double*)malloc(sizeof(double) * (size_t)(rows * 8 * nq)); /* 8 per vector */

    int steps = opts->search_steps > 0 ? opts->search_steps : 12;
    int b = opts->prob_bits > 0 ? opts->prob_bits : (opts->target_bpp <= 7.0 ? 11 : 12);
    if (b < 9 || b > 15) {
        free(norms); free(srows); free(sfields); free(ys); epo_free(bl);
        return -1;
    }
    double s = 1.0;
    for (;;) {
        /* Geometric search at precision b (§3.4, C.1: 12 steps on [1e-3, 8]). */
        double lo = 1e-3, hi = 8.0;
        for (int it = 0; it < steps; ++it) {
            s = sqrt(lo * hi);
            double rate = estimate_rate(&sh, W, norms, srows, rs, s, b, sfields);
            if (rate > opts->target_bpp) lo = s;
            else hi = s;
        }
        s = sqrt(lo * hi);
        for (int64_t r = 0; r < rows; ++r)
            quantize_row(W + r * cols, cols, norms[r], s, sh.direct_z8, bl->fields + NFIELDS * nq * r, ys + r * 8 * nq);
        table_t tabs[MAX_TABLES];
        uint64_t amax = count_tables(bl->fields, sh.nvec, sh.pooled, sh.ntab, 0, tabs);
        for (int t = 0; t < sh.ntab; ++t) table_free(&tabs[t]);
        if (amax <= (1u << b)) break;
        if (b < 15) {
            b += 1; /* C.1: raise b and repeat the scale selection */
            continue;
        }
        /* C.1: at the maximum precision, coarsen s <- 1.05 s A_max / 2^b until it fits. */
        while (amax > (1u << b)) {
            s = 1.05 * s * (double)amax / (double)(1u << b);
            for (int64_t r = 0; r < rows; ++r)
                quantize_row(W + r * cols, cols, norms[r], s, sh.direct_z8, bl->fields + NFIELDS * nq * r,
                             ys + r * 8 * nq);
            amax = count_tables(bl->fields, sh.nvec, sh.pooled, sh.ntab, 0, tabs);
            for (int t = 0; t < sh.ntab; ++t) table_free(&tabs[t]);
        }
        break;
    }
    bl->b = b;
    bl->s = s;
    bl->row_scales = (float*)malloc(sizeof(float) * (size_t)rows);
    /* the refit runs over the row's real entries (the padding is not data) */
    for (int64_t r = 0; r < rows; ++r) bl->row_scales[r] = epo_refit_row(W + r * cols, ys + r * 8 * nq, cols);
    if (opts->rdo_candidates > 1)
        rdo_refine(&sh, W, norms, s, b, opts->rdo_candidates, opts->rdo_sweeps > 0 ? opts->rdo_sweeps : 1,
                   bl->fields, bl->row_scales);
    int rc = code_fields(bl, sh.pooled);
    free(norms);
    free(srows);
    free(sfields);
    free(ys);
    if (rc) {
        epo_free(bl);
        return rc;
    }
    *out = bl;
    return 0;
}

/* Size estimate of the search at a given (s, b): exposed for the rate tests. */
double epo_estimate_rate(const float* W, int64_t rows, int64_t cols, const epo_opts* opts, double s, int b) {
    shape_t sh;
    sh.rows = rows;
    sh.cols = cols;
    sh.nvec = rows * ceil_div(cols, 8);
    sh.pooled = opts->pooled != 0;
    sh.direct_z8 = opts->direct_z8 != 0;
    sh.ntab = sh.pooled ? 9 : 17;
    sh.has_container_scales = opts->has_container_scales != 0;
    int64_t V = opts->tile_vectors > 0 ? opts->tile_vectors : epo_tile_vectors(epo_default_tile_symbols(opts->target_bpp));
    sh.ntiles = ceil_div(sh.nvec, V);
    int64_t nq = ceil_div(cols, 8);
    double* norms = (double*)malloc(sizeof(double) * (size_t)rows);
    for (int64_t r = 0; r < rows; ++r) norms[r] = epo_row_norm(W + r * cols, cols);
    int64_t* srows = (int64_t*)malloc(sizeof(int64_t) * (size_t)rows);
    int64_t sv = opts->sample_vectors > 0 ? opts->sample_vectors : (1 << 18);
    int64_t rs = epo_sample_rows(rows, cols, sv, opts->seed, srows);
    int32_t* sfields = (int32_t*)malloc(sizeof(int32_t) * (size_t)(NFIELDS * nq * rs));
    double rate = estimate_rate(&sh, W, norms, srows, rs, s, b, sfields);
    free(norms);
    free(srows);
    free(sfields);
    return rate;
}

/* ------------------------------------------------------------------------ */
/* Accessors (the Python wrapper copies the blob out through these).         */
/* ------------------------------------------------------------------------ */

void epo_blob_info(const epo_blob* bl, int64_t* ints, double* dbls) {
    ints[0] = bl->rows;
    ints[1] = bl->cols;
    ints[2] = bl->nvec;
    ints[3] = bl->b;
    ints[4] = bl->V;
    ints[5] = bl->ntiles;
    ints[6] = bl->payload_words;
    ints[7] = bl->freq_bytes;
    ints[8] = bl->stored_bytes;
    ints[9] = bl->ntab;
    ints[10] = bl->flags;
    dbls[0] = bl->s;
    dbls[1] = bl->stored_bpp;
    dbls[2] = bl->target_bpp;
}

void epo_blob_copy(const epo_blob* bl, uint16_t* payload, uint32_t* tile_index, uint8_t* freq_tables,
                   float* row_scales, int32_t* fields) {
    if (payload) memcpy(payload, bl->payload, sizeof(uint16_t) * (size_t)bl->payload_words);
    if (tile_index) memcpy(tile_index, bl->tile_index, sizeof(uint32_t) * (size_t)(33 * (int64_t)bl->ntiles + 1));
    if (freq_tables) memcpy(freq_tables, bl->freq_tables, (size_t)bl->freq_bytes);
    if (row_scales) memcpy(row_scales, bl->row_scales, sizeof(float) * (size_t)bl->rows);
    if (fields) memcpy(fields, bl->fields, sizeof(int32_t) * (size_t)(NFIELDS * bl->nvec));
}

/* ------------------------------------------------------------------------ */
/* Output dtype conversions, written from the format definitions.           */
/* BF16: 1-8-7 binary; FP16: IEEE binary16 (1-5-10, bias 15, subnormals,    */
/* overflow to inf); FP8 E4M3 (OCP "fn": bias 7, no inf, largest finite     */
/* 448), saturating; INT8: nearest integer, clamped to [-127, 127].          */
/* All round to nearest, ties to even.  READING: the saturating FP8 and the */
/* symmetric INT8 clamp (the pages only say "dtype conversion").            */
/* ------------------------------------------------------------------------ */

static uint32_t f32_bits(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    return u;
}

uint16_t epo_f32_to_bf16(float x) {
    uint32_t u = f32_bits(x);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u); /* NaN */
    uint32_t hi = u >> 16, rem = u & 0xFFFFu;
    if (rem > 0x8000u || (rem == 0x8000u && (hi & 1u))) hi += 1; /* may carry into the exponent: inf */
    return (uint16_t)hi;
}

/* Round |x| (finite, double) to a binary format with m mantissa bits and least normal exponent emin. */
static double round_to_format(double ax, int m, int emin) {
    if (ax == 0.0) return 0.0;
    int e;
    frexp(ax, &e); /* ax = fr * 2^e, fr in [0.5, 1) -> floor(log2 ax) = e - 1 */
    int ex = e - 1;
    if (ex < emin) ex = emin;
    double ulp = ldexp(1.0, ex - m);
    return nearbyint(ax / ulp) * ulp; /* ax/ulp is exact: fp32 values fit in double */
}

uint16_t epo_f32_to_fp16(float x) {
    uint32_t u = f32_bits(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if ((u & 0x7F800000u) == 0x7F800000u) return (u & 0x007FFFFFu) ? (uint16_t)0x7E00u : (uint16_t)(sign | 0x7C00u);
    double ax = fabs((double)x);
    double r = round_to_format(ax, 10, -14);
    if (r >= 65536.0) return (uint16_t)(sign | 0x7C00u); /* beyond 65504 after rounding: inf */
    if (r == 0.0) return sign;
    int e;
    double fr = frexp(r, &e);
    int ex = e - 1;
    if (ex < -14) { /* subnormal: r = n * 2^-24 */
        return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
    }
    uint32_t mant = (uint32_t)((fr * 2.0 - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)((ex + 15) << 10) | (uint16_t)mant);
}

uint8_t epo_f32_to_e4m3(float x) {
    uint32_t u = f32_bits(x);
    uint8_t sign = (uint8_t)((u >> 24) & 0x80u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7F; /* NaN */
    double ax = fabs((double)x);
    if (ax >= 448.0) return (uint8_t)(sign | 0x7E); /* saturate to the largest finite, 448 */
    double r = round_to_format(ax, 3, -6);
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return sign;
    int e;
    double fr = frexp(r, &e);
    int ex = e - 1;
    if (ex < -6) return (uint8_t)(sign | (uint8_t)(r / ldexp(1.0, -9))); /* subnormal: n * 2^-9 */
    uint32_t mant = (uint32_t)((fr * 2.0 - 1.0) * 8.0);
    return (uint8_t)(sign | (uint8_t)((ex + 7) << 3) | (uint8_t)mant);
}

int8_t epo_f32_to_int8(float x) {
    double r = nearbyint((double)x);
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (int8_t)r;
}

/* UINT8 container with its offset ([paper] App. B, Table 6: integer inputs are
 * scaled per tensor before the cast, the unsigned container carrying an offset,
 * which the error figures subtract again).  Reading: the codec codes
 * the container's codes minus 128, and the decoder adds the 128 back: the
 * nearest integer (ties to even), clamped to [-128, 127], plus 128. */
uint8_t epo_f32_to_uint8(float x) {
    double r = nearbyint((double)x);
    if (r > 127.0) r = 127.0;
    if (r < -128.0) r = -128.0;
    return (uint8_t)(r + 128.0);
}

/* dtype codes shared with the Python wrapper of the oracle */
enum { EPO_BF16 = 0, EPO_FP16 = 1, EPO_E4M3 = 2, EPO_INT8 = 3, EPO_FP32 = 4, EPO_LATTICE = 5, EPO_UINT8 = 6 };

static int dtype_size(int dt) {
    switch (dt) {
        case EPO_BF16: case EPO_FP16: return 2;
        case EPO_E4M3: case EPO_INT8: case EPO_UINT8: return 1;
        case EPO_FP32: case EPO_LATTICE: return 4;
        default: return 0;
    }
}

void epo_convert(const float* in, int64_t n, int dtype, void* out) {
    for (int64_t i = 0; i < n; ++i) {
        switch (dtype) {
            case EPO_BF16: ((uint16_t*)out)[i] = epo_f32_to_bf16(in[i]); break;
            case EPO_FP16: ((uint16_t*)out)[i] = epo_f32_to_fp16(in[i]); break;
            case EPO_E4M3: ((uint8_t*)out)[i] = epo_f32_to_e4m3(in[i]); break;
            case EPO_INT8: ((int8_t*)out)[i] = epo_f32_to_int8(in[i]); break;
            case EPO_UINT8: ((uint8_t*)out)[i] = epo_f32_to_uint8(in[i]); break;
            case EPO_FP32: ((float*)out)[i] = in[i]; break;
            default: break;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Decoder (§3.1 "The decoding path reverses these operations", App. C.3).   */
/* Reads only the four stored buffers: payload, tile index, tables, scales.  */
/* ------------------------------------------------------------------------ */

typedef struct {
    int b, V, ntiles, ntab, flags;
    int64_t rows, cols, nvec;
    int32_t min[MAX_TABLES];
    uint32_t A[MAX_TABLES];
    uint32_t* freq[MAX_TABLES];
    uint32_t* cum[MAX_TABLES];
    int32_t* lut[MAX_TABLES]; /* slot -> symbol index, -1 for an unassigned slot (App. C.3 decoder LUTs) */
} dmodel_t;

static void dmodel_free(dmodel_t* m) {
    for (int t = 0; t < MAX_TABLES; ++t) {
        free(m->freq[t]);
        free(m->cum[t]);
        free(m->lut[t]);
    }
}

/* Parse and check the table header; build the slot -> symbol lookup tables. */
static int dmodel_load(const uint8_t* ft, int64_t rows, int64_t cols, dmodel_t* m) {
    memset(m, 0, sizeof(*m));
    if (get_u32(ft) != MAGIC || get_u32(ft + 4) != 1) return -5;
    m->b = (int)get_u32(ft + 8);
    m->V = (int)get_u32(ft + 12);
    if (get_u32(ft + 16) != J_LANES) return -5;
    m->ntiles = (int)get_u32(ft + 20);
    m->rows = (int64_t)get_u64(ft + 24);
    m->cols = (int64_t)get_u64(ft + 32);
    m->ntab = (int)get_u32(ft + 40);
    m->flags = (int)get_u32(ft + 44);
    if (m->b < 9 || m->b > 15 || m->V < 1) return -5;
    if (m->rows != rows || m->cols != cols) return -5;
    if (!((m->ntab == 17 && !(m->flags & 2)) || (m->ntab == 9 && (m->flags & 2)))) return -5;
    m->nvec = rows * ceil_div(cols, 8);
    if (m->ntiles != ceil_div(m->nvec, m->V)) return -5;
    uint32_t M = 1u << m->b;
    int64_t o = header_bytes(m->ntab);
    for (int t = 0; t < m->ntab; ++t) {
        m->min[t] = (int32_t)get_u32(ft + HDR_FIXED + 8 * t);
        m->A[t] = get_u32(ft + HDR_FIXED + 8 * t + 4);
        if (m->A[t] > M) return -5;
        m->freq[t] = (uint32_t*)calloc(m->A[t] + 1, sizeof(uint32_t));
        m->cum[t] = (uint32_t*)calloc(m->A[t] + 1, sizeof(uint32_t));
        m->lut[t] = (int32_t*)malloc(sizeof(int32_t) * M);
        for (uint32_t s = 0; s < M; ++s) m->lut[t][s] = -1;
        uint64_t sum = 0;
        for (uint32_t s = 0; s < m->A[t]; ++s) {
            m->freq[t][s] = get_u16(ft + o);
            o += 2;
            m->cum[t][s] = (uint32_t)sum;
            sum += m->freq[t][s];
        }
        if (m->A[t] && sum != M) return -5;
        for (uint32_t s = 0; s < m->A[t]; ++s)
            for (uint32_t k = 0; k < m->freq[t][s]; ++k) m->lut[t][m->cum[t][s] + k] = (int32_t)s;
    }
    return 0;
}

/*
 * Decode the fields of tiles [t0, t1).  fields_out receives 9 values per
 * vector, starting with the first vector of tile t0.  Returns 0, or -5 when
 * the stream is inconsistent (a word read past the tile's end, an unassigned
 * slot, a terminal state other than 2^15, or a cursor that misses the next
 * tile's offset).
 */
static int decode_tiles_fields(const dmodel_t* m, const uint16_t* payload, const uint32_t* tix, int64_t t0,
                               int64_t t1, int32_t* fields_out) {
    uint32_t M = 1u << m->b;
    int pooled = (m->flags & 2) != 0;
    int64_t total = tix[33 * (int64_t)m->ntiles];
    for (int64_t t = t0; t < t1; ++t) {
        int64_t v0 = t * m->V;
        int64_t vt = m->nvec - v0 < m->V ? m->nvec - v0 : m->V;
        int64_t cur = tix[33 * t], end = tix[33 * t + 33];
        if (cur > end || end > total) return -5;
        uint64_t x[J_LANES];
        for (int j = 0; j < J_LANES; ++j) {
            x[j] = tix[33 * t + 1 + j];
            if (x[j] < STATE_LOW || x[j] >= (1ull << 31)) return -5;
        }
        int64_t rounds = ceil_div(vt, J_LANES);
        for (int64_t step = 0; step < NFIELDS * rounds; ++step) {
            int64_t r = step / NFIELDS;
            int fld = (int)(step % NFIELDS);
            for (int j = 0; j < J_LANES; ++j) {
                int64_t v = J_LANES * r + j;
                if (v >= vt) continue;
                int32_t* f = fields_out + NFIELDS * (v0 - t0 * m->V + v);
                int tb = table_of(fld, fld == 0 ? 0 : f[0], pooled);
                if (m->A[tb] == 0) return -5;
                uint32_t slot = (uint32_t)(x[j] & (M - 1));
                int32_t sym = m->lut[tb][slot];
                if (sym < 0) return -5;
                x[j] = (uint64_t)m->freq[tb][sym] * (x[j] >> m->b) + slot - m->cum[tb][sym];
                if (x[j] < STATE_LOW) {
                    if (cur >= end) return -5;
                    x[j] = (x[j] << 16) | payload[cur++];
                }
                f[fld] = sym + m->min[tb];
            }
        }
        for (int j = 0; j < J_LANES; ++j)
            if (x[j] != STATE_LOW) return -5;
        if (cur != end) return -5;
    }
    return 0;
}

int epo_decode_fields(const uint16_t* payload, const uint32_t* tile_index, const uint8_t* freq_tables,
                      int64_t rows, int64_t cols, int64_t t0, int64_t t1, int32_t* fields_out) {
    dmodel_t m;
    int rc = dmodel_load(freq_tables, rows, cols, &m);
    if (!rc) {
        if (t0 < 0 || t1 > m.ntiles || t0 > t1) rc = -1;
        else rc = decode_tiles_fields(&m, payload, tile_index, t0, t1, fields_out);
    }
    dmodel_free(&m);
    return rc;
}

/*
 * Decode tiles [t0, t1) to dtype: fields -> 2y (App. A.3 inverse) ->
 * w = fl32(sigma_row * y) (one FP32 multiply; y is exact in FP32) -> dtype.
 * out receives the tiles' weights contiguously (8 per vector), starting with
 * the first weight of tile t0.  EPO_LATTICE writes 2y as int32.
 */
int epo_decode(const uint16_t* payload, const uint32_t* tile_index, const uint8_t* freq_tables,
               const float* row_scales, int64_t rows, int64_t cols, int dtype, int64_t t0, int64_t t1, void* out) {
    dmodel_t m;
    int rc = dmodel_load(freq_tables, rows, cols, &m);
    if (rc) {
        dmodel_free(&m);
        return rc;
    }
    if (t0 < 0 || t1 > m.ntiles || t0 > t1 || dtype_size(dtype) == 0) {
        dmodel_free(&m);
        return -1;
    }
    int64_t v0 = t0 * m.V;
    int64_t v1 = t1 * (int64_t)m.V < m.nvec ? t1 * (int64_t)m.V : m.nvec;
    int64_t nv = v1 - v0;
    int32_t* fields = (int32_t*)malloc(sizeof(int32_t) * (size_t)(NFIELDS * (nv > 0 ? nv : 1)));
    rc = decode_tiles_fields(&m, payload, tile_index, t0, t1, fields);
    int direct = (m.flags & 1) != 0;
    /* vector v holds elements row * cols + 8q .. (row = v / nq, q = v % nq) up to the row's
     * end; the vectors [v0, v1) cover the contiguous element range [E(v0), E(v1)) */
    int64_t nq = ceil_div(cols, 8);
    int64_t e0 = (v0 / nq) * cols + 8 * (v0 % nq);
    int sz = dtype_size(dtype);
    for (int64_t i = 0; !rc && i < nv; ++i) {
        int64_t f[NFIELDS], y2[8];
        for (int k = 0; k < NFIELDS; ++k) f[k] = fields[NFIELDS * i + k];
        epo_point_from_fields(f, direct, y2);
        int64_t row = (v0 + i) / nq, q = (v0 + i) % nq;
        float sigma = row_scales[row];
        uint8_t* o = (uint8_t*)out + (size_t)(row * cols + 8 * q - e0) * (size_t)sz;
        for (int k = 0; k < 8 && 8 * q + k < cols; ++k) {
            if (dtype == EPO_LATTICE) {
                ((int32_t*)o)[k] = (int32_t)y2[k];
                continue;
            }
            float yk = (float)((double)y2[k] * 0.5); /* exact */
            float w = sigma * yk;                     /* the single FP32 multiply */
            epo_convert(&w, 1, dtype, o + (size_t)k * (size_t)sz);
        }
    }
    free(fields);
    dmodel_free(&m);
    return rc;
}
