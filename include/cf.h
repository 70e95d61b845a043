/*
 * cf.h -- C ABI of the B200 residual-compression library (libcf.so).
 *
 * The library implements residual compression with error feedback of the
 * per-step activations that parallel diffusion inference exchanges, as
 * described in "Accelerating Parallel Diffusion Model Serving with Residual
 * Compression" (NeurIPS 2025 paper notes):
 *   - "Overall framework": each step sends the compressed residual
 *     D_t = a_t - ahat_{t-1} instead of a_t; the receiver rebuilds
 *     ahat_t = ahat_{t-1} + C(D_t).
 *   - "Key design: error feedback": the part of the residual that was not
 *     sent, e_t = D_t - C(D_t), is kept by the sender and added to the next
 *     residual: D_t = a_t - ahat_{t-1} + e_{t-1}.
 *   - "Key design: residual compression" / experiments table: 1-bit (16x)
 *     and 2-bit (8x) quantisation of the residual.
 *   - "Key design: system co-design": an N:M block sparsifier instead of a
 *     global TopK.
 *   - "Key design: low-rank strategy": X ~ U V^T by warm-started subspace
 *     iteration, U and V quantised to INT4.
 *   - "Limitations": the first step has no history and is sent in full.
 * The pages fix no bit layout, scale or rounding rule; the ones below are
 * this library's definition (see the payload layout section).
 *
 * Conventions for every entry point
 *   - Returns an int status: CF_OK (0) or a negative CF_ERR_* code.  No C++
 *     exception crosses the ABI.  cf_strerror() names a code.
 *   - "device" pointers are CUDA device memory of the current device; "host"
 *     pointers are ordinary host memory.  The caller owns every pointer it
 *     passes; the library never frees caller memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Encode/decode are asynchronous on that stream; the state's
 *     step counter advances when the call is enqueued.
 *   - A state is used by one host thread and one stream at a time.
 *   - Kernels never trap, never spin and never read out of bounds: argument
 *     errors are rejected on the host before any launch, and a payload that
 *     does not match the receiver (mode, shape, step) is detected on the
 *     device, leaves the receiver untouched and is reported by cf_status().
 *
 * Tensor layout: an activation tensor is row-major [rows][cols] (rows =
 * tokens, cols = channels), 16-byte aligned, row pitch = cols elements.  A
 * batch of B equally shaped tensors is either one contiguous
 * [B][rows][cols] array (cf_encode / cf_decode) or B separate tensors given
 * by a host array of device pointers (cf_encode_batched / cf_decode_batched).
 *
 * Payload layout (little-endian; every section starts 16-byte aligned):
 *   header, 64 bytes:
 *     0 u32 magic 0x31504643 ("CFP1") | 4 u32 mode | 8 u32 flags (bit0 = warm-up)
 *    12 u32 dtype | 16 u64 step | 24 u64 rows | 32 u64 cols | 40 u32 batch
 *    44 u32 p0 | 48 u32 p1 | 52 u32 ef | 56 u32 p2 | 60 u32 0
 *     (p0,p1,p2) = (N, M, 0) for CF_NM, (rank, int4 flag, iterations) for
 *     CF_LOWRANK, zero otherwise.
 *   then one body per tensor, tensor-major, each padded to 16 bytes:
 *     warm-up   : the raw activation [rows][cols] in the activation dtype
 *     CF_IDENTITY: D as fp32 [rows][cols]
 *     CF_SIGN1  : scale bf16 [rows] (pad 16) | bits u32 [rows][cols/32];
 *                 bit (i mod 32) of word i/32 is 1 iff D_i < 0;
 *                 C_i = bit ? -S : +S with S = bf16(fp32(mean_i |D_i|)),
 *                 the mean taken as an exact fixed-point sum (order
 *                 independent): E = floor(log2 max|D|), q_i =
 *                 floor(|D_i| 2^(31-E)), mean = fp64(sum q_i) 2^(E-31) / cols
 *     CF_Q2     : scale bf16 [rows] (pad 16) | codes u32 [rows][cols/16];
 *                 code of column i in bits 2(i mod 16).. of word i/16;
 *                 S = bf16(max |D|), u = (D/S)*1.5 + 1.5 clamped to [0,3],
 *                 q = round-half-even(u), C = ((2q-3) S)/3
 *     CF_NM     : values bf16 [rows][cols/M][N] (pad 16) |
 *                 indices u32 [rows][(cols/M) N log2(M) / 32];
 *                 per block of M columns the N largest |D| (lower index wins
 *                 ties), kept indices ascending; field j of a row (log2 M
 *                 bits, LSB first) is block j/N's (j mod N)-th index
 *     CF_LOWRANK: (int4) scales fp32 sU[r], sV[r] (pad 16) | U nibbles
 *                 [rows*r] (pad 16) | V nibbles [cols*r] (pad 16); element
 *                 (i,k) is nibble i*r+k, low nibble first, two's complement
 *                 in [-7,7]; C = sum_k (qU_ik sU_k)(qV_jk sV_k).
 *                 (fp32 factors) U fp32 [rows][r] (pad 16) | V fp32 [cols][r]
 *   All fp32 arithmetic of the recurrence is IEEE round-to-nearest-even
 *   without contraction: D = (a - ahat) + e, e = D - C, ahat = ahat + C.
 */
#ifndef CF_H_
#define CF_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CF_API __attribute__((visibility("default")))
#else
#define CF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define CF_OK 0
#define CF_ERR_ARG (-1)          /* NULL or out-of-range argument */
#define CF_ERR_SHAPE (-2)        /* rows/cols/batch violate the mode's shape rule */
#define CF_ERR_ROLE (-3)         /* encode on a receiver state or decode on a sender state */
#define CF_ERR_UNSUPPORTED (-4)  /* valid request this build does not implement */
#define CF_ERR_CUDA (-5)         /* a CUDA runtime call or kernel launch failed */
#define CF_ERR_NOMEM (-6)        /* device allocation failed or workspace too small */
#define CF_ERR_DESYNC (-7)       /* (device) payload header did not match the receiver */
#define CF_ERR_ALIGN (-8)        /* a pointer is not 16-byte aligned */
#define CF_ERR_STATE (-9)        /* handle is not a live state (destroyed or foreign) */
#define CF_ERR_SIZE (-10)        /* a host buffer size does not match */
#define CF_ERR_TIMEOUT (-11)     /* (device) a bounded wait for an asynchronous copy gave up */
#define CF_ERR_TOO_LARGE (-12)   /* problem larger than the allocation-free entry point's fixed scratch */

/* ---- enumerations ---------------------------------------------------- */
/* CF_BLOCKSEL is Otil's selective transmission ("Informative sub-block
 * selection", "Dynamic round-robin"): not a residual codec.  The rows are a
 * token grid bs_grid_h x (rows / bs_grid_h) in raster order, cut into
 * bs_block x bs_block blocks spanning all channels; each selective step sends
 * the bs_k blocks whose cosine dissimilarity d = 1 - <x_{t-1}, x_t>_F /
 * (||x_{t-1}|| ||x_t||) against the previous activation is largest, among the
 * blocks not yet sent in the current round (ties: lower block index; a block
 * with all values unchanged has d = 0, one with exactly one zero norm d = 1);
 * the round restarts once every block has been sent; the receiver keeps
 * every other block as last received.  The first bs_warm steps are sent in
 * full.  Error feedback does not apply (ef is ignored). */
typedef enum { CF_IDENTITY = 0, CF_SIGN1 = 1, CF_Q2 = 2, CF_NM = 3, CF_LOWRANK = 4, CF_BLOCKSEL = 5 } cf_mode;
typedef enum { CF_F32 = 0, CF_BF16 = 1 } cf_dtype;
typedef enum { CF_SENDER = 0, CF_RECEIVER = 1 } cf_role;
/* Error-feedback form ("Key design: error feedback"):
 *   CF_EF_EXPLICIT  D = (a - ahat) + e   (default; the recurrence as stated)
 *   CF_EF_IMPLICIT  D = a - ahat; e = D - C is still recorded.
 *   CF_EF_OFF       residual compression without error feedback, the
 *                   variant whose error the page says grows linearly with
 *                   the step count: the sender's ahat slot holds fp32 of the
 *                   previous activation, D = a_t - a_{t-1}, and the sender's
 *                   update is ahat = fp32(a_t); e is neither read nor
 *                   written.  The receiver is the same for all three. */
typedef enum { CF_EF_EXPLICIT = 0, CF_EF_IMPLICIT = 1, CF_EF_OFF = 2 } cf_ef;

/* which tensor cf_tensor() returns */
typedef enum { CF_T_RECON = 0, CF_T_ERROR = 1, CF_T_VPREV = 2 } cf_which;

/* Creation parameters.  Fill with cf_params_init() and override fields. */
typedef struct {
    int dtype;                 /* cf_dtype of the activations (and recon, warm-up payload) */
    int role;                  /* cf_role */
    int ef;                    /* cf_ef */
    int nm_n, nm_m;            /* CF_NM: M in {4,16}; N in {1,2}, N < M */
    int rank;                  /* CF_LOWRANK: 1 <= rank <= min(rows, cols, 128) */
    int iters;                 /* CF_LOWRANK: subspace-iteration sweeps per step, 1 or 2 */
    int lr_int4;               /* CF_LOWRANK: 1 = INT4 factors, 0 = fp32 factors */
    int batch;                 /* >= 1 equally shaped tensors per step */
    uint64_t seed;             /* CF_LOWRANK: seed of the first step's V */
    void *workspace;           /* optional caller-owned device memory for the state, or NULL */
    size_t workspace_bytes;    /* its size; must be >= cf_workspace_bytes() */
    int bs_grid_h;             /* CF_BLOCKSEL: token-grid height; 0 = square grid (rows a square) */
    int bs_block;              /* CF_BLOCKSEL: block side in tokens, 4, 8 or 16 (default 8) */
    int bs_k;                  /* CF_BLOCKSEL: blocks per step, 1..K; 0 = K/4 ("k/K = 1/4") */
    int bs_warm;               /* CF_BLOCKSEL: leading steps sent in full, >= 1 (default 5) */
    int state_dtype;           /* CF_F32 (default): ahat and e in fp32.  CF_BF16: the bf16-state
                                  option of the streaming modes with bf16 activations -- every
                                  state update rounds to bf16 (nearest even), on both sides
                                  alike; state traffic 8 instead of 16 bytes per element */
    double lr_qr2_tol;         /* CF_LOWRANK: the second CholeskyQR pass uses the first-order
                                  factor of Q1^T Q1 when every entry of Q1^T Q1 - I is at most
                                  this (orthogonality error about 3 rank tol^2 per entry);
                                  0 = always the full elimination; 0 <= tol <= 2^-12
                                  (default 2^-16) */
} cf_params;

typedef struct cf_state cf_state;

/* Library version string (static storage). */
CF_API const char *cf_version(void);

/* Human-readable name of a status code (static storage; never NULL). */
CF_API const char *cf_strerror(int status);

/* Defaults: bf16, sender, explicit EF, N:M 2:16, rank 70, 1 sweep, INT4,
 * batch 1, seed 0, no workspace, block selection 8x8 blocks with k = K/4 and
 * 5 full steps, fp32 state, lr_qr2_tol 2^-16.  Returns CF_ERR_ARG if p is NULL. */
CF_API int cf_params_init(cf_params *p);

/* Device bytes a state of this configuration needs (state tensors, status
 * word, and for CF_LOWRANK the factor scratch).  *out receives the size. */
CF_API int cf_workspace_bytes(int64_t rows, int64_t cols, int mode, const cf_params *p, size_t *out);

/* Create a sender or receiver state on the current CUDA device.  Shape
 * rules: rows >= 1; cols % 8 == 0 and cols <= 8192; CF_SIGN1 cols % 32 == 0;
 * CF_Q2 cols % 16 == 0; CF_NM cols % M == 0 and (cols/M) N log2(M) % 32 == 0;
 * CF_BLOCKSEL: the grid and both of its sides divisible by bs_block,
 * K = (H/b)(W/b) <= 4096 blocks, batch 1;
 * CF_LOWRANK rows % 128 == 0, cols % 128 == 0, rank <= min(rows, cols, 128),
 * (rows + cols) * round_up(rank, 64) < 2^31 (32-bit factor indices),
 * batch 1 (the low-rank state also holds its factor scratch: about
 * 8 rows*cols bytes for a sender).  The state owns its tensors (in `workspace`
 * when given, else in memory it allocates with cudaMalloc) and starts at
 * step 0 (the warm-up step).  Blocks until its memory is initialised. */
CF_API int cf_create(int64_t rows, int64_t cols, int mode, const cf_params *p, cf_state **out);

/* Bytes of the payload the next call writes: warmup != 0 for step 0 (raw
 * activations), 0 for every later step. */
CF_API int cf_payload_bytes(const cf_state *s, int warmup, size_t *out);

/* Sender step ("Overall framework" + "error feedback"): reads the device
 * activations a ([batch][rows][cols], contiguous, state dtype), writes the
 * device payload (cf_payload_bytes(s, step == 0) bytes), and updates the
 * sender's ahat and e in place.  One fused kernel per call for the
 * streaming modes.  Asynchronous on `stream`.  CF_LOWRANK: the launch chain
 * is captured on a stream the state owns and run as one CUDA graph on
 * `stream` (the state keeps the executable graph and updates it in place
 * each call); when `stream` is itself being captured, the kernels are
 * recorded into the caller's graph instead. */
CF_API int cf_encode(cf_state *s, const void *a, void *payload, void *stream);

/* Receiver step: reads the device payload, updates the receiver's ahat and
 * writes the device reconstruction recon = cast(ahat) ([batch][rows][cols],
 * state dtype).  A header mismatch sets the device status (see cf_status)
 * and leaves ahat and recon untouched.  Asynchronous on `stream`. */
CF_API int cf_decode(cf_state *s, const void *payload, void *recon, void *stream);

/* As cf_encode / cf_decode for `batch` separate tensors: a_ptrs / recon_ptrs
 * are HOST arrays of `batch` device pointers (read during the call only).
 * Every tensor of the step is handled by one launch.  batch <= 1024. */
CF_API int cf_encode_batched(cf_state *s, const void *const *a_ptrs, void *payload, void *stream);
CF_API int cf_decode_batched(cf_state *s, const void *payload, void *const *recon_ptrs, void *stream);

/* Synchronises `stream`, then returns the state's sticky device status:
 * CF_OK; CF_ERR_DESYNC after a payload that did not match this receiver;
 * CF_ERR_TIMEOUT if a kernel's bounded wait for one of its own asynchronous
 * copies gave up (the kernel then returned early; its outputs are not valid).
 * Returns CF_ERR_CUDA if the stream reports an error. */
CF_API int cf_status(cf_state *s, void *stream);

/* Device pointer and byte size of a state tensor (fp32, [batch][rows][cols];
 * CF_T_RECON is ahat of this role, CF_T_ERROR is e (sender), CF_T_VPREV is
 * the low-rank warm start [batch][cols][rank] (sender)). */
CF_API int cf_tensor(cf_state *s, int which, void **dptr, size_t *bytes);

/* Steps already enqueued on this state (0 before the warm-up step). */
CF_API int cf_step(const cf_state *s, uint64_t *out);

/* Start a new request: the next call is the warm-up step again; the status
 * is cleared.  Synchronous (device memset on the legacy stream). */
CF_API int cf_reset(cf_state *s);

/* Test hook for the failure detection of the low-rank kernels (the pages
 * have no counterpart: this is the library's own bounded-wait check).  With
 * polls > 0, every later reconstruction launch of this CF_LOWRANK state (the
 * receiver's decode; the last kernel of a sender's encode) issues none of its
 * operand copies and waits at most `polls` polls for them, so its bounded
 * wait gives up: the kernel records the timeout in the state's status word
 * (cf_status then returns CF_ERR_TIMEOUT), frees its tensor memory and
 * returns without writing ahat, e or recon.  No copy or MMA is left in
 * flight.  In a sender's encode the orthonormalisation kernel's first
 * grid-wide barrier is made to run out as well (one block withholds its
 * arrival; every block waits at most `polls` polls, records the timeout and
 * returns before Q is formed, so the payload's U scales stay zero).
 * polls = 0 restores normal operation; cf_reset clears the status.
 * Returns CF_ERR_UNSUPPORTED for the other modes. */
CF_API int cf_test_wait_timeout(cf_state *s, uint32_t polls);

/* Checkpoint / resume: cf_state_bytes gives the host buffer size;
 * cf_state_export copies the state (step, status and tensors) into it,
 * cf_state_import restores a state of the same configuration.  Both
 * synchronise `stream`. */
CF_API int cf_state_bytes(const cf_state *s, size_t *out);
CF_API int cf_state_export(const cf_state *s, void *host, size_t bytes, void *stream);
CF_API int cf_state_import(cf_state *s, const void *host, size_t bytes, void *stream);

/* Allocation-free low-rank decode.  The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory at decode
 * time -- code that runs where cudaMalloc is unavailable or forbidden (inside
 * a framework that owns every allocation, a fixed-memory serving process, a
 * library call made from a stream callback or capture-sensitive code path).
 * It decodes one steady-state low-rank payload exactly as cf_decode does on
 * a CF_LOWRANK receiver (same kernels, bit-identical ahat and recon), but
 * with no state object and no allocation: the caller passes the receiver's
 * reconstruction `ahat` (device fp32 [rows][cols], updated in place), the
 * output `recon` (device, [rows][cols] in p->dtype), a device status word
 * `status` (int; the kernels OR in 1 when the payload header does not match
 * rows, cols, p and `step`, leaving ahat and recon untouched, and 2 when a
 * bounded wait gave up), the device `payload` and the stream.  p supplies
 * dtype, ef, rank, iters and lr_int4 (role, batch and workspace are
 * ignored: this decode always handles one tensor).  `step` (>= 1) is the
 * step the payload must carry; the warm-up step (raw activations) is not
 * handled here.
 * The dequantised factors go to a fixed scratch array of 8 MiB that every
 * GPU loading the library holds until exit: (rows*kp*(int4 ? 2 : 4) +
 * cols*kp*4) bytes, each part rounded up to 256, must fit, where kp is rank
 * rounded up to 64; larger problems return CF_ERR_TOO_LARGE.  The first call
 * on a device looks up that array's device address and sets kernel
 * attributes, so make it before any stream capture.  All calls share the
 * one array: calls whose work overlaps on the GPU (other streams, other
 * threads) race; serialise them.  Shape rules as for CF_LOWRANK. */
CF_API int cf_lowrank_decode_noalloc(int64_t rows, int64_t cols, const cf_params *p, uint64_t step,
                                     const void *payload, float *ahat, void *recon, int *status, void *stream);

/* Free the state (and its memory, unless it lives in a caller workspace).
 * Synchronises the device first.  Later calls with the handle return
 * CF_ERR_STATE. */
CF_API int cf_destroy(cf_state *s);

#ifdef __cplusplus
}
#endif

#endif /* CF_H_ */
