/*
 * cf_oracle.c -- plain, slow CPU oracle for residual compression with error
 * feedback (CompactFusion).  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the benchmark's CPU-baseline leg load it; the product path never
 * does.  It shares no code, header, table or helper with the CUDA library.
 *
 * Source: "Accelerating Parallel Diffusion Model Serving with Residual
 * Compression" (NeurIPS 2025 paper notes), sections "Overall framework",
 * "Key design: residual compression", "Key design: error feedback",
 * "Key design: low-rank strategy for extreme ratios" and "Limitations"
 * (first step is sent in full).
 *
 * What is computed, per tensor, per step (explicit error feedback):
 *   step 0 :  payload = a_0 (raw), ahat_S = ahat_R = fp32(a_0), e = 0
 *   step t :  D = (a_t - ahat_S) + e          (fp32, two RN operations)
 *             payload = enc(D);  C = dec(payload)
 *             e = D - C;  ahat_S = ahat_S + C  (fp32 RN)
 *   receiver: ahat_R = ahat_R + dec(payload);  recon = cast(ahat_R)
 * With implicit error feedback D = a_t - ahat_S (the error already lives in
 * the reconstruction) and e is only recorded.  Without error feedback (the
 * variant whose error the page says grows linearly with the step count) the
 * sender's ahat slot holds fp32(a_{t-1}): D = a_t - a_{t-1}, and the update
 * is ahat_S = fp32(a_t); e stays zero.
 *
 * The pages give no bit layouts, scales or rounding rules.  The encodings
 * below are the readings this project fixes (IEEE round-to-nearest-even in
 * fp32, no contraction; compile with -ffp-contract=off):
 *   SIGN1 : bit = (D < 0); C = bit ? -S : +S; S = bf16(mean|D|) where the
 *           mean is an exact fixed-point sum (see sign1_scale).
 *   Q2    : S = bf16(max|D|); u = (D/S)*1.5 + 1.5 clamped to [0,3];
 *           q = rint(u); C = ((2q-3)*S)/3.
 *   NM    : per block of M columns keep the N largest |D| (lower index wins
 *           ties); values bf16(D); indices log2(M)-bit nibbles.
 *   LOWRANK: warm-started subspace iteration Y = D V, Q = orth(Y),
 *           V = D^T Q, computed in fp64 with Householder QR; U = Q and V
 *           are quantised to INT4 per column.
 *   IDENTITY: payload = D (fp32), C = D.
 *
 *   BLOCKSEL: Otil's selective transmission ("Informative sub-block
 *           selection", "Dynamic round-robin"): the token grid H x W (rows =
 *           H*W in raster order) is cut into b x b blocks (all channels); per
 *           step the k blocks of largest cosine dissimilarity against the
 *           previous activation, among the blocks not yet sent this round,
 *           are sent raw; the round restarts once every block has been sent.
 *
 * Parity pins live in tests/test_oracle_*.py; every function here is checked
 * there against brute force, closed forms or a library routine.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_IDENTITY 0
#define ORC_SIGN1 1
#define ORC_Q2 2
#define ORC_NM 3
#define ORC_LOWRANK 4
#define ORC_BLOCKSEL 5 /* Otil-style block selection (second workload) */

#define ORC_F32 0
#define ORC_BF16 1

#define ORC_EF_EXPLICIT 0
#define ORC_EF_IMPLICIT 1
#define ORC_EF_OFF 2 /* residual against the previous activation, no feedback */

#define ORC_MAGIC 0x31504643u /* bytes 'C','F','P','1' */
#define ORC_HDR 64

/* ------------------------------------------------------------------ */
/* scalar helpers                                                      */
/* ------------------------------------------------------------------ */

static uint32_t f2u(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }
static float u2f(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }

/* bfloat16 round-to-nearest-even, by definition: the two bf16 neighbours of
 * x (sign-magnitude bit patterns) are the truncation and the next pattern
 * away from zero; pick the nearer, on a tie the one with an even last bit.
 * NaN maps to a quiet NaN with the same sign. */
uint16_t orc_bf16_from_f32(float x)
{
    uint32_t u = f2u(x);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lo = u & 0xffff0000u;          /* toward zero */
    uint32_t rem = u & 0x0000ffffu;
    uint32_t pick;
    if (rem < 0x8000u) pick = lo;
    else if (rem > 0x8000u) pick = lo + 0x10000u;
    else pick = ((lo >> 16) & 1u) ? lo + 0x10000u : lo;
    return (uint16_t)(pick >> 16);
}

float orc_f32_from_bf16(uint16_t h) { return u2f((uint32_t)h << 16); }

static int ilog2_i(int m)
{
    int c = 0;
    while ((1 << c) < m) c++;
    return c;
}

static size_t pad16(size_t b) { return (b + 15u) & ~(size_t)15u; }

/* ------------------------------------------------------------------ */
/* per-row statistics                                                  */
/* ------------------------------------------------------------------ */

/* SIGN1 scale: bf16(fp32(mean |d_i|)).  The mean is made independent of the
 * summation order by summing exact fixed-point values with 31 fraction bits
 * below the row maximum's leading bit:
 *   m = max|d|; if m == 0 the scale is 0
 *   E = floor(log2 m), F = 31
 *   q_i = floor(|d_i| * 2^(F-E))   (exact: a 24-bit significand scaled by a
 *                                   power of two, then floored; q_i < 2^32)
 *   Q = sum q_i in uint64           (exact for n < 2^32)
 *   mean = fp64(Q) * 2^(E-F) / n    (fp64 round-to-nearest; Q < 2^53 is exact)
 * The truncation moves the mean by less than 2^(E-F) <= n 2^-31 of itself.
 * The L2-optimal scale for sign codes is mean|d| (argmin_s sum (d - s sgn d)^2). */
#define ORC_SIGN1_F 31
uint16_t orc_sign1_scale(const float *d, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(d[i]);
        if (a > m) m = a;
    }
    if (m == 0.0f) return 0;
    int k;
    frexp((double)m, &k);                 /* m = f * 2^k, f in [0.5, 1) */
    int E = k - 1;
    int F = ORC_SIGN1_F;
    uint64_t Q = 0;
    for (int64_t i = 0; i < n; i++) {
        double s = ldexp((double)fabsf(d[i]), F - E);
        Q += (uint64_t)floor(s);
    }
    double mean = ldexp((double)Q, E - F) / (double)n;
    return orc_bf16_from_f32((float)mean);
}

/* Q2 scale: bf16(max |d_i|) -- a max is order-free. */
uint16_t orc_q2_scale(const float *d, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(d[i]);
        if (a > m) m = a;
    }
    return orc_bf16_from_f32(m);
}

/* Q2 code of one element, for scale S (fp32 value of the bf16 scale). */
int orc_q2_code(float d, float S)
{
    if (S == 0.0f) return 0;
    float t = d / S;
    t = t * 1.5f;
    float u = t + 1.5f;
    if (u < 0.0f) u = 0.0f;
    if (u > 3.0f) u = 3.0f;
    return (int)rintf(u);                 /* current rounding mode: nearest-even */
}

/* Q2 reconstruction level q in {0,1,2,3}: ((2q-3) * S) / 3  = {-S,-S/3,S/3,S}. */
float orc_q2_level(int q, float S)
{
    float num = (float)(2 * q - 3) * S;
    return num / 3.0f;
}

/* N:M selection in one block of m values: the n indices with the largest
 * |d|, the lower index winning ties, returned in ascending order. */
void orc_nm_select(const float *d, int m, int n, int *idx_out)
{
    int taken[64];
    for (int j = 0; j < m; j++) taken[j] = 0;
    for (int s = 0; s < n; s++) {
        int best = -1;
        for (int j = 0; j < m; j++) {
            if (taken[j]) continue;
            if (best < 0 || fabsf(d[j]) > fabsf(d[best])) best = j;
        }
        taken[best] = 1;
    }
    int c = 0;
    for (int j = 0; j < m; j++)
        if (taken[j]) idx_out[c++] = j;
}

/* splitmix64 (Steele, Lea, Flood 2014; Vigna's public-domain reference): one
 * output for a 64-bit state value x: advance by the golden gamma, then mix. */
uint64_t orc_splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

/* Initial right factor for the first low-rank step (the pages leave it
 * open): V0[j,k] = 2 * (splitmix64(seed ^ (j*r + k)) >> 40) * 2^-24 - 1,
 * uniform in [-1, 1) and exact in fp32. */
float orc_lr_v0(uint64_t seed, int64_t j, int r, int k)
{
    uint64_t z = orc_splitmix64(seed ^ (uint64_t)(j * (int64_t)r + k));
    double u = (double)(z >> 40) * (1.0 / 16777216.0);
    return (float)(2.0 * u - 1.0);
}

/* ------------------------------------------------------------------ */
/* state                                                               */
/* ------------------------------------------------------------------ */

typedef struct {
    int64_t rows, cols;
    int mode, dtype, ef;
    int nm_n, nm_m;
    int rank, iters, lr_int4;
    int batch;
    uint64_t seed;
    float *ahat_s;   /* [batch][rows][cols] sender reconstruction */
    float *err;      /* [batch][rows][cols] error-feedback memory */
    float *ahat_r;   /* [batch][rows][cols] receiver reconstruction */
    float *vprev;    /* LOWRANK: [batch][cols][rank] fp32 warm start */
    int bs_h, bs_w, bs_b, bs_k, bs_warm, bs_K; /* BLOCKSEL grid, block side, blocks per step */
    uint8_t *bs_sent; /* BLOCKSEL: [K] 1 = sent in the current round */
    int state_bf16;   /* the bf16-state option: every state update rounds to bf16 */
    int vprev_valid;
    uint64_t step_s, step_r;
    int status;      /* 0 ok; nonzero after a header mismatch */
} orc_state;

static int64_t elems(const orc_state *o) { return o->rows * o->cols; }

static size_t act_size(int dtype) { return dtype == ORC_BF16 ? 2u : 4u; }

/* body bytes of one tensor's steady-state payload */
size_t orc_tensor_body_bytes(const orc_state *o)
{
    int64_t R = o->rows, Cc = o->cols;
    switch (o->mode) {
    case ORC_IDENTITY: return pad16((size_t)(R * Cc) * 4u);
    case ORC_SIGN1: return pad16((size_t)R * 2u) + pad16((size_t)(R * Cc / 8));
    case ORC_Q2: return pad16((size_t)R * 2u) + pad16((size_t)(R * Cc / 4));
    case ORC_NM: {
        int64_t blocks = Cc / o->nm_m;
        int64_t bits = blocks * o->nm_n * ilog2_i(o->nm_m);
        int64_t words = (bits + 31) / 32;
        return pad16((size_t)(R * blocks * o->nm_n) * 2u) + pad16((size_t)(R * words) * 4u);
    }
    case ORC_LOWRANK:
        if (o->lr_int4)
            return pad16((size_t)o->rank * 8u) + pad16((size_t)((R * o->rank + 1) / 2)) +
                   pad16((size_t)((Cc * o->rank + 1) / 2));
        return pad16((size_t)(R * o->rank) * 4u) + pad16((size_t)(Cc * o->rank) * 4u);
    case ORC_BLOCKSEL:
        return pad16((size_t)o->bs_k * 4u) +
               (size_t)o->bs_k * (size_t)o->bs_b * (size_t)o->bs_b * (size_t)Cc * act_size(o->dtype);
    }
    return 0;
}

/* number of leading steps sent in full */
static uint64_t warm_steps(const orc_state *o) { return o->mode == ORC_BLOCKSEL ? (uint64_t)o->bs_warm : 1u; }

/* 1 if the next encode (receiver: decode) is a full-size warm-up step */
int orc_next_is_warm(const orc_state *o, int receiver)
{
    return (receiver ? o->step_r : o->step_s) < warm_steps(o);
}

size_t orc_payload_bytes(const orc_state *o, int warmup)
{
    size_t body = warmup ? pad16((size_t)elems(o) * act_size(o->dtype)) : orc_tensor_body_bytes(o);
    return ORC_HDR + body * (size_t)o->batch;
}

orc_state *orc_create(int64_t rows, int64_t cols, int mode, int dtype, int ef, int nm_n, int nm_m,
                      int rank, int iters, int lr_int4, int batch, uint64_t seed)
{
    if (rows < 1 || cols < 1 || batch < 1) return NULL;
    if (mode < ORC_IDENTITY || mode > ORC_BLOCKSEL) return NULL;
    if (dtype != ORC_F32 && dtype != ORC_BF16) return NULL;
    if (ef != ORC_EF_EXPLICIT && ef != ORC_EF_IMPLICIT && ef != ORC_EF_OFF) return NULL;
    if (cols % 8) return NULL;
    if (mode == ORC_SIGN1 && cols % 32) return NULL;
    if (mode == ORC_Q2 && cols % 16) return NULL;
    if (mode == ORC_NM) {
        if (nm_m != 4 && nm_m != 8 && nm_m != 16) return NULL;
        if (nm_n < 1 || nm_n >= nm_m || cols % nm_m) return NULL;
    }
    if (mode == ORC_LOWRANK) {
        if (rank < 1 || rank > rows || rank > cols || iters < 1) return NULL;
    }
    orc_state *o = (orc_state *)calloc(1, sizeof(orc_state));
    o->rows = rows; o->cols = cols; o->mode = mode; o->dtype = dtype; o->ef = ef;
    o->nm_n = nm_n; o->nm_m = nm_m; o->rank = rank; o->iters = iters; o->lr_int4 = lr_int4;
    o->batch = batch; o->seed = seed;
    size_t n = (size_t)(rows * cols) * (size_t)batch;
    o->ahat_s = (float *)calloc(n, 4);
    o->err = (float *)calloc(n, 4);
    o->ahat_r = (float *)calloc(n, 4);
    if (mode == ORC_LOWRANK) o->vprev = (float *)calloc((size_t)cols * rank * batch, 4);
    return o;
}

void orc_destroy(orc_state *o)
{
    if (!o) return;
    free(o->ahat_s); free(o->err); free(o->ahat_r); free(o->vprev); free(o->bs_sent);
    free(o);
}

uint64_t orc_step(const orc_state *o, int receiver) { return receiver ? o->step_r : o->step_s; }
int orc_status(const orc_state *o) { return o->status; }

/* Threads of the row-parallel loops for the calling thread's later calls
 * (timing only: every parallel loop writes disjoint rows, so the results do
 * not depend on it).  Returns the thread count now in effect. */
int orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* which: 0 ahat_S, 1 e, 2 ahat_R, 3 V_prev.  Copies the whole batch. */
float *orc_buffer(orc_state *o, int which)
{
    switch (which) {
    case 0: return o->ahat_s;
    case 1: return o->err;
    case 2: return o->ahat_r;
    case 3: return o->vprev;
    }
    return NULL;
}

void orc_set_vprev_valid(orc_state *o, int v) { o->vprev_valid = v; }

/* BLOCKSEL configuration (required before the first step): token grid
 * h x (rows / h), block side b, k blocks per step, `warm` leading steps sent
 * in full.  Returns 0, or -1 if the grid is not cut evenly into blocks, k is
 * out of range or the state is not a single-tensor BLOCKSEL state. */
int orc_set_blocksel(orc_state *o, int h, int b, int k, int warm)
{
    if (o->mode != ORC_BLOCKSEL || o->batch != 1) return -1;
    if (h < 1 || b < 1 || warm < 1 || o->rows % h) return -1;
    int w = (int)(o->rows / h);
    if (h % b || w % b) return -1;
    int K = (h / b) * (w / b);
    if (k < 1 || k > K) return -1;
    o->bs_h = h; o->bs_w = w; o->bs_b = b; o->bs_k = k; o->bs_warm = warm; o->bs_K = K;
    free(o->bs_sent);
    o->bs_sent = (uint8_t *)calloc((size_t)K, 1);
    return 0;
}

uint8_t *orc_blocksel_sent(orc_state *o) { return o->bs_sent; }

/* The bf16-state option (streaming modes, bf16 activations): ahat_S, e and
 * ahat_R are rounded to bf16 (nearest even) after every update, on both
 * sides alike.  Returns 0, or -1 for a configuration without the option. */
int orc_set_state_bf16(orc_state *o, int on)
{
    if (on && (o->dtype != ORC_BF16 || o->mode == ORC_LOWRANK || o->mode == ORC_BLOCKSEL)) return -1;
    o->state_bf16 = on ? 1 : 0;
    return 0;
}

/* the state's storage rounding */
static float st_round(const orc_state *o, float x)
{
    return o->state_bf16 ? orc_f32_from_bf16(orc_bf16_from_f32(x)) : x;
}
void orc_set_step(orc_state *o, uint64_t s_send, uint64_t s_recv) { o->step_s = s_send; o->step_r = s_recv; }

static float load_act(const void *a, int dtype, int64_t i)
{
    if (dtype == ORC_BF16) return orc_f32_from_bf16(((const uint16_t *)a)[i]);
    return ((const float *)a)[i];
}

static void store_act(void *dst, int dtype, int64_t i, float v)
{
    if (dtype == ORC_BF16) ((uint16_t *)dst)[i] = orc_bf16_from_f32(v);
    else ((float *)dst)[i] = v;
}

static void write_u32(uint8_t *p, uint32_t v) { memcpy(p, &v, 4); }
static void write_u64(uint8_t *p, uint64_t v) { memcpy(p, &v, 8); }

/* 64-byte payload header (little-endian):
 *   0 magic | 4 mode | 8 flags (bit0 warm-up) | 12 dtype | 16 step (u64)
 *  24 rows (u64) | 32 cols (u64) | 40 batch | 44 p0 | 48 p1 | 52 ef | 56 p2 | 60 zero
 *  p0/p1/p2: NM -> N, M, 0; LOWRANK -> rank, int4 flag, iterations;
 *  BLOCKSEL -> grid height, block side, blocks per step; else 0. */
static void write_header(const orc_state *o, uint8_t *p, int warm, uint64_t step)
{
    memset(p, 0, ORC_HDR);
    write_u32(p + 0, ORC_MAGIC);
    write_u32(p + 4, (uint32_t)o->mode);
    write_u32(p + 8, warm ? 1u : 0u);
    write_u32(p + 12, (uint32_t)o->dtype);
    write_u64(p + 16, step);
    write_u64(p + 24, (uint64_t)o->rows);
    write_u64(p + 32, (uint64_t)o->cols);
    write_u32(p + 40, (uint32_t)o->batch);
    uint32_t p0 = 0, p1 = 0, p2 = 0;
    if (o->mode == ORC_NM) { p0 = (uint32_t)o->nm_n; p1 = (uint32_t)o->nm_m; }
    if (o->mode == ORC_LOWRANK) { p0 = (uint32_t)o->rank; p1 = (uint32_t)o->lr_int4; p2 = (uint32_t)o->iters; }
    if (o->mode == ORC_BLOCKSEL) { p0 = (uint32_t)o->bs_h; p1 = (uint32_t)o->bs_b; p2 = (uint32_t)o->bs_k; }
    write_u32(p + 44, p0);
    write_u32(p + 48, p1);
    write_u32(p + 52, (uint32_t)o->ef);
    write_u32(p + 56, p2);
}

static int check_header(const orc_state *o, const uint8_t *p, int warm, uint64_t step)
{
    uint8_t want[ORC_HDR];
    write_header(o, want, warm, step);
    return memcmp(want, p, ORC_HDR) == 0;
}

/* ------------------------------------------------------------------ */
/* streaming modes: per-row encode / decode                            */
/* ------------------------------------------------------------------ */

/* Encode one row's residual d[0..cols) into the payload sections of that
 * row, and return the reconstruction C[0..cols) the payload stands for. */
static void encode_row(const orc_state *o, const float *d, uint8_t *body, int64_t r, float *C)
{
    int64_t n = o->cols, R = o->rows;
    if (o->mode == ORC_IDENTITY) {
        float *pay = (float *)body + r * n;
        for (int64_t i = 0; i < n; i++) { pay[i] = d[i]; C[i] = d[i]; }
    } else if (o->mode == ORC_SIGN1) {
        uint16_t *scales = (uint16_t *)body;
        uint32_t *words = (uint32_t *)(body + pad16((size_t)R * 2u)) + r * (n / 32);
        uint16_t sb = orc_sign1_scale(d, n);
        scales[r] = sb;
        float S = orc_f32_from_bf16(sb);
        for (int64_t w = 0; w < n / 32; w++) words[w] = 0;
        for (int64_t i = 0; i < n; i++) {
            int bit = d[i] < 0.0f;
            if (bit) words[i / 32] |= 1u << (i % 32);
            C[i] = bit ? -S : S;
        }
    } else if (o->mode == ORC_Q2) {
        uint16_t *scales = (uint16_t *)body;
        uint32_t *words = (uint32_t *)(body + pad16((size_t)R * 2u)) + r * (n / 16);
        uint16_t sb = orc_q2_scale(d, n);
        scales[r] = sb;
        float S = orc_f32_from_bf16(sb);
        for (int64_t w = 0; w < n / 16; w++) words[w] = 0;
        for (int64_t i = 0; i < n; i++) {
            int q = orc_q2_code(d[i], S);
            words[i / 16] |= (uint32_t)q << (2 * (i % 16));
            C[i] = orc_q2_level(q, S);
        }
    } else if (o->mode == ORC_NM) {
        int M = o->nm_m, N = o->nm_n, lb = ilog2_i(M);
        int64_t blocks = n / M;
        int64_t words_per_row = (blocks * N * lb + 31) / 32;
        uint16_t *vals = (uint16_t *)body + r * blocks * N;
        uint32_t *idxw = (uint32_t *)(body + pad16((size_t)(R * blocks * N) * 2u)) + r * words_per_row;
        for (int64_t w = 0; w < words_per_row; w++) idxw[w] = 0;
        for (int64_t i = 0; i < n; i++) C[i] = 0.0f;
        int idx[64];
        for (int64_t b = 0; b < blocks; b++) {
            orc_nm_select(d + b * M, M, N, idx);
            for (int s = 0; s < N; s++) {
                int64_t col = b * M + idx[s];
                uint16_t vb = orc_bf16_from_f32(d[col]);
                vals[b * N + s] = vb;
                C[col] = orc_f32_from_bf16(vb);
                int64_t slot = b * N + s;             /* field number within the row */
                int64_t bit = slot * lb;
                idxw[bit / 32] |= (uint32_t)idx[s] << (bit % 32);
            }
        }
    }
}

/* Rebuild one row's C from the payload (receiver side). */
static void decode_row(const orc_state *o, const uint8_t *body, int64_t r, float *C)
{
    int64_t n = o->cols, R = o->rows;
    if (o->mode == ORC_IDENTITY) {
        const float *pay = (const float *)body + r * n;
        for (int64_t i = 0; i < n; i++) C[i] = pay[i];
    } else if (o->mode == ORC_SIGN1) {
        const uint16_t *scales = (const uint16_t *)body;
        const uint32_t *words = (const uint32_t *)(body + pad16((size_t)R * 2u)) + r * (n / 32);
        float S = orc_f32_from_bf16(scales[r]);
        for (int64_t i = 0; i < n; i++) C[i] = ((words[i / 32] >> (i % 32)) & 1u) ? -S : S;
    } else if (o->mode == ORC_Q2) {
        const uint16_t *scales = (const uint16_t *)body;
        const uint32_t *words = (const uint32_t *)(body + pad16((size_t)R * 2u)) + r * (n / 16);
        float S = orc_f32_from_bf16(scales[r]);
        for (int64_t i = 0; i < n; i++) {
            int q = (int)((words[i / 16] >> (2 * (i % 16))) & 3u);
            C[i] = orc_q2_level(q, S);
        }
    } else if (o->mode == ORC_NM) {
        int M = o->nm_m, N = o->nm_n, lb = ilog2_i(M);
        int64_t blocks = n / M;
        int64_t words_per_row = (blocks * N * lb + 31) / 32;
        const uint16_t *vals = (const uint16_t *)body + r * blocks * N;
        const uint32_t *idxw = (const uint32_t *)(body + pad16((size_t)(R * blocks * N) * 2u)) + r * words_per_row;
        for (int64_t i = 0; i < n; i++) C[i] = 0.0f;
        for (int64_t b = 0; b < blocks; b++)
            for (int s = 0; s < N; s++) {
                int64_t bit = (b * N + s) * lb;
                int j = (int)((idxw[bit / 32] >> (bit % 32)) & (uint32_t)(M - 1));
                C[b * M + j] = orc_f32_from_bf16(vals[b * N + s]);
            }
    }
}

/* ------------------------------------------------------------------ */
/* low-rank: subspace iteration in fp64                                 */
/* ------------------------------------------------------------------ */

/* Thin QR of Y (m x r, row-major) by Householder reflections, in fp64.
 * Returns Q (m x r, row-major, orthonormal columns) and diag(R), with the
 * sign convention diag(R) >= 0 (Q's column k is negated when R_kk < 0).
 * Columns whose |R_kk| <= tol * |R_00| are rank-deficient; their Q column
 * is set to zero and dead[k] = 1. */
void orc_householder_qr(const double *Y, int64_t m, int r, double tol, double *Q, double *rdiag, int *dead)
{
    double *A = (double *)malloc(sizeof(double) * (size_t)m * r);
    double *V = (double *)calloc((size_t)m * r, sizeof(double)); /* reflectors, column k in V[:,k] */
    double *beta = (double *)calloc((size_t)r, sizeof(double));
    memcpy(A, Y, sizeof(double) * (size_t)m * r);
    for (int k = 0; k < r; k++) {
        double nrm = 0.0;
        for (int64_t i = k; i < m; i++) nrm += A[i * r + k] * A[i * r + k];
        nrm = sqrt(nrm);
        double x0 = A[(int64_t)k * r + k];
        double alpha = (x0 >= 0.0) ? -nrm : nrm;   /* R_kk = alpha */
        rdiag[k] = alpha;
        if (nrm == 0.0) { beta[k] = 0.0; continue; }
        for (int64_t i = k; i < m; i++) V[i * r + k] = A[i * r + k];
        V[(int64_t)k * r + k] -= alpha;
        double vn = 0.0;
        for (int64_t i = k; i < m; i++) vn += V[i * r + k] * V[i * r + k];
        beta[k] = (vn > 0.0) ? 2.0 / vn : 0.0;
        /* apply H_k = I - beta v v^T to the remaining columns */
        for (int c = k; c < r; c++) {
            double s = 0.0;
            for (int64_t i = k; i < m; i++) s += V[i * r + k] * A[i * r + c];
            s *= beta[k];
            for (int64_t i = k; i < m; i++) A[i * r + c] -= s * V[i * r + k];
        }
    }
    /* Q = H_0 H_1 ... H_{r-1} applied to the first r columns of I */
    for (int64_t i = 0; i < m; i++)
        for (int c = 0; c < r; c++) Q[i * r + c] = (i == c) ? 1.0 : 0.0;
    for (int k = r - 1; k >= 0; k--) {
        if (beta[k] == 0.0) continue;
        for (int c = 0; c < r; c++) {
            double s = 0.0;
            for (int64_t i = k; i < m; i++) s += V[i * r + k] * Q[i * r + c];
            s *= beta[k];
            for (int64_t i = k; i < m; i++) Q[i * r + c] -= s * V[i * r + k];
        }
    }
    double r00 = fabs(rdiag[0]);
    for (int k = 0; k < r; k++) {
        dead[k] = fabs(rdiag[k]) <= tol * r00;
        double sg = rdiag[k] < 0.0 ? -1.0 : 1.0;
        for (int64_t i = 0; i < m; i++) Q[i * r + k] = dead[k] ? 0.0 : sg * Q[i * r + k];
        rdiag[k] = fabs(rdiag[k]);
    }
    free(A); free(V); free(beta);
}

/* Symmetric per-column INT4 quantisation of X (m x r): s_k = fp32(absmax_k/7);
 * code = clamp(rint(x / s_k), -7, 7); a zero column gets s_k = 0, codes 0. */
static void int4_quantise(const double *X, int64_t m, int r, float *scale, int8_t *code)
{
    for (int k = 0; k < r; k++) {
        double amax = 0.0;
        for (int64_t i = 0; i < m; i++) if (fabs(X[i * r + k]) > amax) amax = fabs(X[i * r + k]);
        float s = (float)(amax / 7.0);
        scale[k] = s;
        for (int64_t i = 0; i < m; i++) {
            int q = 0;
            if (s != 0.0f) {
                double t = rint(X[i * r + k] / (double)s);
                if (t > 7.0) t = 7.0;
                if (t < -7.0) t = -7.0;
                q = (int)t;
            }
            code[i * r + k] = (int8_t)q;
        }
    }
}

static void put_nibble(uint8_t *base, int64_t idx, int q)
{
    uint8_t v = (uint8_t)(q & 0xF);
    if (idx & 1) base[idx / 2] = (uint8_t)((base[idx / 2] & 0x0F) | (v << 4));
    else base[idx / 2] = (uint8_t)((base[idx / 2] & 0xF0) | v);
}

static int get_nibble(const uint8_t *base, int64_t idx)
{
    int v = (idx & 1) ? (base[idx / 2] >> 4) : (base[idx / 2] & 0xF);
    return (v & 0x8) ? v - 16 : v;
}

/* Dequantised factors from a low-rank tensor body: U (rows x r), V (cols x r), fp64. */
static void lr_factors_from_body(const orc_state *o, const uint8_t *body, double *U, double *V)
{
    int64_t R = o->rows, Cc = o->cols;
    int r = o->rank;
    if (o->lr_int4) {
        const float *sU = (const float *)body;
        const float *sV = sU + r;
        const uint8_t *cu = body + pad16((size_t)r * 8u);
        const uint8_t *cv = cu + pad16((size_t)((R * r + 1) / 2));
        for (int64_t i = 0; i < R; i++)
            for (int k = 0; k < r; k++) U[i * r + k] = (double)get_nibble(cu, i * r + k) * (double)sU[k];
        for (int64_t j = 0; j < Cc; j++)
            for (int k = 0; k < r; k++) V[j * r + k] = (double)get_nibble(cv, j * r + k) * (double)sV[k];
    } else {
        const float *u = (const float *)body;
        const float *v = (const float *)(body + pad16((size_t)(R * r) * 4u));
        for (int64_t i = 0; i < R * r; i++) U[i] = u[i];
        for (int64_t i = 0; i < Cc * r; i++) V[i] = v[i];
    }
}

/* C = U V^T (rows x cols), each entry rounded once to fp32. */
static void lr_reconstruct(const orc_state *o, const double *U, const double *V, float *C)
{
    int64_t R = o->rows, Cc = o->cols;
    int r = o->rank;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < R; i++)
        for (int64_t j = 0; j < Cc; j++) {
            double s = 0.0;
            for (int k = 0; k < r; k++) s += U[i * r + k] * V[j * r + k];
            C[i * Cc + j] = (float)s;
        }
}

/* One tensor's low-rank encode: d (rows x cols fp32) -> body; writes C. */
static void lowrank_encode(orc_state *o, const float *d, float *vprev, uint8_t *body, float *C)
{
    int64_t R = o->rows, Cc = o->cols;
    int r = o->rank;
    double *V = (double *)malloc(sizeof(double) * (size_t)Cc * r);
    double *Y = (double *)malloc(sizeof(double) * (size_t)R * r);
    double *Q = (double *)malloc(sizeof(double) * (size_t)R * r);
    double *rd = (double *)malloc(sizeof(double) * (size_t)r);
    int *dead = (int *)malloc(sizeof(int) * (size_t)r);
    /* warm start: previous step's V; the first step, and any all-zero
     * column, takes the seeded draw V0. */
    for (int k = 0; k < r; k++) {
        int zero = 1;
        if (o->vprev_valid)
            for (int64_t j = 0; j < Cc; j++) if (vprev[j * r + k] != 0.0f) { zero = 0; break; }
        for (int64_t j = 0; j < Cc; j++)
            V[j * r + k] = zero ? (double)orc_lr_v0(o->seed, j, r, k) : (double)vprev[j * r + k];
    }
    for (int it = 0; it < o->iters; it++) {
        /* Y = D V */
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < R; i++)
            for (int k = 0; k < r; k++) {
                double s = 0.0;
                for (int64_t j = 0; j < Cc; j++) s += (double)d[i * Cc + j] * V[j * r + k];
                Y[i * r + k] = s;
            }
        orc_householder_qr(Y, R, r, 1e-6, Q, rd, dead);
        /* V = D^T Q */
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < Cc; j++)
            for (int k = 0; k < r; k++) {
                double s = 0.0;
                for (int64_t i = 0; i < R; i++) s += (double)d[i * Cc + j] * Q[i * r + k];
                V[j * r + k] = s;
            }
    }
    for (int64_t i = 0; i < Cc * r; i++) vprev[i] = (float)V[i];
    o->vprev_valid = 1;
    memset(body, 0, orc_tensor_body_bytes(o));
    if (o->lr_int4) {
        float *sU = (float *)body;
        float *sV = sU + r;
        uint8_t *cu = body + pad16((size_t)r * 8u);
        uint8_t *cv = cu + pad16((size_t)((R * r + 1) / 2));
        int8_t *code = (int8_t *)malloc((size_t)(R > Cc ? R : Cc) * r);
        int4_quantise(Q, R, r, sU, code);
        for (int64_t i = 0; i < R * r; i++) put_nibble(cu, i, code[i]);
        int4_quantise(V, Cc, r, sV, code);
        for (int64_t i = 0; i < Cc * r; i++) put_nibble(cv, i, code[i]);
        free(code);
    } else {
        float *u = (float *)body;
        float *v = (float *)(body + pad16((size_t)(R * r) * 4u));
        for (int64_t i = 0; i < R * r; i++) u[i] = (float)Q[i];
        for (int64_t i = 0; i < Cc * r; i++) v[i] = (float)V[i];
    }
    double *Ud = (double *)malloc(sizeof(double) * (size_t)R * r);
    double *Vd = (double *)malloc(sizeof(double) * (size_t)Cc * r);
    lr_factors_from_body(o, body, Ud, Vd);
    lr_reconstruct(o, Ud, Vd, C);
    free(Ud); free(Vd);
    free(V); free(Y); free(Q); free(rd); free(dead);
}

/* ------------------------------------------------------------------ */
/* public entry points                                                 */
/* ------------------------------------------------------------------ */

/* Sender step: a = [batch][rows][cols] in the state's dtype; payload gets
 * orc_payload_bytes(o, step==0) bytes.  Returns 0. */
/* ------------------------------------------------------------------ */
/* block selection                                                     */
/* ------------------------------------------------------------------ */

#define ORC_BS_NONE 0xffffffffu /* index of an unused payload slot */

/* token (row) index of element (y, x) of block i */
static int64_t bs_token(const orc_state *o, int i, int y, int x)
{
    int nbx = o->bs_w / o->bs_b;
    int by = i / nbx, bx = i % nbx;
    return (int64_t)(by * o->bs_b + y) * o->bs_w + bx * o->bs_b + x;
}

/* Cosine dissimilarity of block i between the previous activation p and the
 * current one a ("Informative sub-block selection"): d = 1 - <p, a>_F /
 * (||p||_F ||a||_F), the Frobenius sums over the block's tokens in raster
 * order and all channels, in fp64 (each product of two fp32 values is exact).
 * Readings for the cases the formula leaves open: a block whose values are
 * all unchanged has d = 0; a block with exactly one zero norm has d = 1. */
static double bs_dissimilarity(const orc_state *o, int i, const float *p, const float *a)
{
    double dot = 0.0, np_ = 0.0, na = 0.0;
    int changed = 0;
    for (int y = 0; y < o->bs_b; y++)
        for (int x = 0; x < o->bs_b; x++) {
            int64_t t = bs_token(o, i, y, x);
            for (int64_t c = 0; c < o->cols; c++) {
                double u = p[t * o->cols + c], v = a[t * o->cols + c];
                if (u != v) changed = 1;
                dot += u * v;
                np_ += u * u;
                na += v * v;
            }
        }
    if (!changed) return 0.0;
    if (np_ == 0.0 || na == 0.0) return 1.0;
    return 1.0 - dot / (sqrt(np_) * sqrt(na));
}

typedef struct { double d; int i; } bs_cand;

/* larger dissimilarity first; on equal dissimilarity the lower block index */
static int bs_cmp(const void *x, const void *y)
{
    const bs_cand *a = (const bs_cand *)x, *b = (const bs_cand *)y;
    if (a->d > b->d) return -1;
    if (a->d < b->d) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

static int bs_cmp_index(const void *x, const void *y)
{
    int a = *(const int *)x, b = *(const int *)y;
    return (a > b) - (a < b);
}

/* One selective step: the top-k of the unsent blocks ("Dynamic round-robin":
 * selection only from the blocks not yet sent this round; when every block
 * has been sent the round restarts), their raw values in ascending block
 * order, unused slots (the last step of a round may have fewer than k
 * blocks left) marked ORC_BS_NONE and zero.  The sender's state becomes
 * fp32(a_t). */
static void blocksel_encode(orc_state *o, const void *a, uint8_t *body)
{
    int K = o->bs_K, k = o->bs_k, b = o->bs_b;
    int64_t E = elems(o);
    float *cur = (float *)malloc(sizeof(float) * (size_t)E);
    for (int64_t i = 0; i < E; i++) cur[i] = load_act(a, o->dtype, i);
    bs_cand *cand = (bs_cand *)malloc(sizeof(bs_cand) * (size_t)K);
    int nc = 0;
    for (int i = 0; i < K; i++)
        if (!o->bs_sent[i]) {
            cand[nc].d = bs_dissimilarity(o, i, o->ahat_s, cur);
            cand[nc].i = i;
            nc++;
        }
    qsort(cand, (size_t)nc, sizeof(bs_cand), bs_cmp);
    int m = nc < k ? nc : k;
    int *sel = (int *)malloc(sizeof(int) * (size_t)(m > 0 ? m : 1));
    for (int j = 0; j < m; j++) sel[j] = cand[j].i;
    qsort(sel, (size_t)m, sizeof(int), bs_cmp_index);
    size_t asz = act_size(o->dtype);
    size_t blk = (size_t)b * b * (size_t)o->cols * asz;
    uint8_t *data = body + pad16((size_t)k * 4u);
    memset(body, 0, orc_tensor_body_bytes(o));
    for (int j = 0; j < k; j++) write_u32(body + 4 * j, j < m ? (uint32_t)sel[j] : ORC_BS_NONE);
    for (int j = 0; j < m; j++)
        for (int y = 0; y < b; y++)
            for (int x = 0; x < b; x++) {
                int64_t t = bs_token(o, sel[j], y, x);
                memcpy(data + (size_t)j * blk + ((size_t)y * b + x) * (size_t)o->cols * asz,
                       (const uint8_t *)a + (size_t)t * (size_t)o->cols * asz, (size_t)o->cols * asz);
            }
    for (int j = 0; j < m; j++) o->bs_sent[sel[j]] = 1;
    int all = 1;
    for (int i = 0; i < K; i++) all &= o->bs_sent[i];
    if (all) memset(o->bs_sent, 0, (size_t)K);
    memcpy(o->ahat_s, cur, sizeof(float) * (size_t)E);
    free(cur); free(cand); free(sel);
}

/* Receiver side: the sent blocks replace the receiver's values; every other
 * block keeps the value it last received. */
static void blocksel_decode(orc_state *o, const uint8_t *body)
{
    int K = o->bs_K, k = o->bs_k, b = o->bs_b;
    size_t asz = act_size(o->dtype);
    size_t blk = (size_t)b * b * (size_t)o->cols * asz;
    const uint8_t *data = body + pad16((size_t)k * 4u);
    for (int j = 0; j < k; j++) {
        uint32_t i;
        memcpy(&i, body + 4 * j, 4);
        if (i == ORC_BS_NONE || i >= (uint32_t)K) continue;
        for (int y = 0; y < b; y++)
            for (int x = 0; x < b; x++) {
                int64_t t = bs_token(o, (int)i, y, x);
                const uint8_t *src = data + (size_t)j * blk + ((size_t)y * b + x) * (size_t)o->cols * asz;
                for (int64_t c = 0; c < o->cols; c++) o->ahat_r[t * o->cols + c] = load_act(src, o->dtype, c);
            }
    }
}

int orc_encode(orc_state *o, const void *a, uint8_t *payload)
{
    int64_t E = elems(o);
    int warm = o->step_s < warm_steps(o);
    if (o->mode == ORC_BLOCKSEL && !o->bs_sent) return -1;
    write_header(o, payload, warm, o->step_s);
    uint8_t *body0 = payload + ORC_HDR;
    if (warm) {
        size_t tb = pad16((size_t)E * act_size(o->dtype));
        for (int b = 0; b < o->batch; b++) {
            uint8_t *body = body0 + tb * b;
            memset(body, 0, tb);
            memcpy(body, (const uint8_t *)a + (size_t)E * act_size(o->dtype) * b, (size_t)E * act_size(o->dtype));
            for (int64_t i = 0; i < E; i++) {
                o->ahat_s[(int64_t)b * E + i] = load_act(a, o->dtype, (int64_t)b * E + i);
                o->err[(int64_t)b * E + i] = 0.0f;
            }
        }
        o->step_s++;
        return 0;
    }
    size_t tb = orc_tensor_body_bytes(o);
    if (o->mode == ORC_BLOCKSEL) {
        blocksel_encode(o, a, body0);
        o->step_s++;
        return 0;
    }
    float *d = (float *)malloc(sizeof(float) * (size_t)E);
    float *C = (float *)malloc(sizeof(float) * (size_t)E);
    for (int b = 0; b < o->batch; b++) {
        float *ah = o->ahat_s + (int64_t)b * E;
        float *er = o->err + (int64_t)b * E;
        uint8_t *body = body0 + tb * b;
        if (o->mode != ORC_LOWRANK) memset(body, 0, tb);
        for (int64_t i = 0; i < E; i++) {
            float x = load_act(a, o->dtype, (int64_t)b * E + i);
            float t = x - ah[i];
            d[i] = (o->ef == ORC_EF_EXPLICIT) ? t + er[i] : t;
        }
        if (o->mode == ORC_LOWRANK) {
            lowrank_encode(o, d, o->vprev + (int64_t)b * o->cols * o->rank, body, C);
        } else {
            #pragma omp parallel for schedule(static)
            for (int64_t r = 0; r < o->rows; r++) encode_row(o, d + r * o->cols, body, r, C + r * o->cols);
        }
        for (int64_t i = 0; i < E; i++) {
            if (o->ef == ORC_EF_OFF) {
                /* "Key design: error feedback" names what happens without
                 * feedback: the untransmitted error is dropped, and the
                 * next residual is taken against this step's activation */
                ah[i] = st_round(o, load_act(a, o->dtype, (int64_t)b * E + i));
            } else {
                er[i] = st_round(o, d[i] - C[i]);
                ah[i] = st_round(o, ah[i] + C[i]);
            }
        }
    }
    free(d); free(C);
    o->step_s++;
    return 0;
}

/* Receiver step: rebuilds ahat_R from the payload and writes recon =
 * cast(ahat_R) ([batch][rows][cols] in the state's dtype).  A header that
 * does not match this receiver's expectation (mode, shape, step, ...) sets
 * status = 1 and leaves ahat_R and recon untouched.  Returns the status. */
int orc_decode(orc_state *o, const uint8_t *payload, void *recon)
{
    int64_t E = elems(o);
    int warm = o->step_r < warm_steps(o);
    if (o->mode == ORC_BLOCKSEL && !o->bs_sent) return -1;
    if (!check_header(o, payload, warm, o->step_r)) {
        o->status = 1;
        o->step_r++;
        return 1;
    }
    const uint8_t *body0 = payload + ORC_HDR;
    if (warm) {
        size_t tb = pad16((size_t)E * act_size(o->dtype));
        for (int b = 0; b < o->batch; b++)
            for (int64_t i = 0; i < E; i++) {
                float x = load_act(body0 + tb * b, o->dtype, i);
                o->ahat_r[(int64_t)b * E + i] = x;
                store_act(recon, o->dtype, (int64_t)b * E + i, x);
            }
        o->step_r++;
        return 0;
    }
    size_t tb = orc_tensor_body_bytes(o);
    if (o->mode == ORC_BLOCKSEL) {
        blocksel_decode(o, body0);
        for (int64_t i = 0; i < E; i++) store_act(recon, o->dtype, i, o->ahat_r[i]);
        o->step_r++;
        return 0;
    }
    float *C = (float *)malloc(sizeof(float) * (size_t)E);
    for (int b = 0; b < o->batch; b++) {
        const uint8_t *body = body0 + tb * b;
        if (o->mode == ORC_LOWRANK) {
            int r = o->rank;
            double *U = (double *)malloc(sizeof(double) * (size_t)o->rows * r);
            double *V = (double *)malloc(sizeof(double) * (size_t)o->cols * r);
            lr_factors_from_body(o, body, U, V);
            lr_reconstruct(o, U, V, C);
            free(U); free(V);
        } else {
            #pragma omp parallel for schedule(static)
            for (int64_t r = 0; r < o->rows; r++) decode_row(o, body, r, C + r * o->cols);
        }
        float *ah = o->ahat_r + (int64_t)b * E;
        for (int64_t i = 0; i < E; i++) {
            ah[i] = st_round(o, ah[i] + C[i]);
            store_act(recon, o->dtype, (int64_t)b * E + i, ah[i]);
        }
    }
    free(C);
    o->step_r++;
    return 0;
}

/* Reconstruction C that a steady-state payload stands for (one tensor b),
 * without touching any state: used by tests that compare payload meaning. */
int orc_payload_meaning(const orc_state *o, const uint8_t *payload, int b, float *C)
{
    if (o->mode == ORC_BLOCKSEL) return -1; /* a selection carries values, not a residual */
    const uint8_t *body = payload + ORC_HDR + orc_tensor_body_bytes(o) * (size_t)b;
    if (o->mode == ORC_LOWRANK) {
        int r = o->rank;
        double *U = (double *)malloc(sizeof(double) * (size_t)o->rows * r);
        double *V = (double *)malloc(sizeof(double) * (size_t)o->cols * r);
        lr_factors_from_body(o, body, U, V);
        lr_reconstruct(o, U, V, C);
        free(U); free(V);
    } else {
        for (int64_t r = 0; r < o->rows; r++) decode_row(o, body, r, C + r * o->cols);
    }
    return 0;
}

/* Low-rank building block exposed for pins: one subspace-iteration sweep
 * sequence on a caller matrix D (m x n fp32), starting from V (n x r fp64,
 * overwritten with the final V); Q (m x r) receives the last orthonormal
 * basis.  No quantisation. */
void orc_subspace_iteration(const float *D, int64_t m, int64_t n, int r, int iters, double *V, double *Q)
{
    double *Y = (double *)malloc(sizeof(double) * (size_t)m * r);
    double *rd = (double *)malloc(sizeof(double) * (size_t)r);
    int *dead = (int *)malloc(sizeof(int) * (size_t)r);
    for (int it = 0; it < iters; it++) {
        for (int64_t i = 0; i < m; i++)
            for (int k = 0; k < r; k++) {
                double s = 0.0;
                for (int64_t j = 0; j < n; j++) s += (double)D[i * n + j] * V[j * r + k];
                Y[i * r + k] = s;
            }
        orc_householder_qr(Y, m, r, 1e-6, Q, rd, dead);
        for (int64_t j = 0; j < n; j++)
            for (int k = 0; k < r; k++) {
                double s = 0.0;
                for (int64_t i = 0; i < m; i++) s += (double)D[i * n + j] * Q[i * r + k];
                V[j * r + k] = s;
            }
    }
    free(Y); free(rd); free(dead);
}

/* BLOCKSEL pin helper: the dissimilarity of every block between two caller
 * activations p and a (fp32 [rows][cols]) into d[K]. */
int orc_blocksel_dissimilarity(const orc_state *o, const float *p, const float *a, double *d)
{
    if (o->mode != ORC_BLOCKSEL || !o->bs_sent) return -1;
    for (int i = 0; i < o->bs_K; i++) d[i] = bs_dissimilarity(o, i, p, a);
    return 0;
}

/* Array helpers for the tests (elementwise, no arithmetic of their own). */
void orc_bf16_from_f32_array(const float *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_bf16_from_f32(x[i]);
}

void orc_f32_from_bf16_array(const uint16_t *h, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_f32_from_bf16(h[i]);
}
