// cf_lowrank.cu -- low-rank mode of libcf on sm_100a.
//
// Method: "Accelerating Parallel Diffusion Model Serving with Residual
// Compression", section "Key design: low-rank strategy for extreme ratios":
// the residual D (with error feedback) is approximated as U V^T by
// warm-started subspace iteration instead of an SVD, and U, V are quantised
// to INT4 so that more rank fits the same bandwidth.  One iteration is
//     Y = D V;  Q = orth(Y);  V = D^T Q          (U = Q is transmitted)
// with V warm-started from the previous step's V.  orth is the thin-QR
// factor with positive diagonal, computed by CholeskyQR2 in fp64 (unique for
// full column rank, so it agrees with a Householder QR up to rounding);
// columns with R_kk <= 1e-6 R_00 are rank deficient and set to zero.
//
// GEMMs: the two thin products (N = rank padded to a multiple of 16) and the
// reconstruction C = U V^T run on the 5th-generation tensor cores (tcgen05
// MMA, operands staged by TMA in 128-byte swizzled K-major tiles, fp32
// accumulators in tensor memory).  Operands are bf16 pairs x = hi + lo
// (hi = bf16(x), lo = bf16(x - hi)), and each product sums hi*hi + hi*lo +
// lo*hi, which keeps about 16 significant bits: enough that the INT4 codes
// the GPU picks agree with an fp64 computation except near rounding ties.
// The reconstruction is one deterministic kernel run by both the sender and
// the receiver on operands dequantised from the payload bytes, so sender and
// receiver reconstructions are bit-identical.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <type_traits>
#include <utility>
#include <mutex>

#include "cf_lowrank.h"
#include "cf_launch.cuh"
#include "cf_umma.cuh"

namespace cfi {
namespace {

constexpr int kTileM = 128;     // UMMA M and TMA box rows of the A operand
constexpr int kTileK = 64;      // bf16 per 128-byte swizzled row
constexpr int kReconN = 128;    // N of a reconstruction tile
constexpr int kStatusDesync = 1;
constexpr int kStatusTimeout = 2;

size_t pad256(size_t b) { return (b + 255u) & ~(size_t)255u; }
size_t pad16(size_t b) { return (b + 15u) & ~(size_t)15u; }

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi)));
}

// Header check for the receiver's kernels (same rule as the streaming decode).
__device__ __forceinline__ bool lr_header_ok(const uint8_t *payload, const Header &expect, int *status) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  if (threadIdx.x < 16) {
    const uint32_t w = reinterpret_cast<const uint32_t *>(payload)[threadIdx.x];
    if (w != expect.w[threadIdx.x]) atomicOr(&bad, 1);
  }
  __syncthreads();
  if (bad) {
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) atomicOr(status, kStatusDesync);
    return false;
  }
  return true;
}

// splitmix64 (Steele, Lea, Flood; Vigna's public-domain reference).
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9e3779b97f4a7c15ull;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}

// First step's V (the pages leave it open): 2 * (splitmix64(seed ^ (j r + k)) >> 40) * 2^-24 - 1.
__device__ __forceinline__ float v0_entry(uint64_t seed, int64_t j, int r, int k) {
  const uint64_t z = splitmix64(seed ^ (uint64_t)(j * (int64_t)r + k));
  const double u = (double)(z >> 40) * (1.0 / 16777216.0);
  return (float)(2.0 * u - 1.0);
}

// ---------------------------------------------------------------- V preparation


// Vt (split bf16, [rp][cols]) from the warm start: the previous step's V
// (fp32 [cols][r]), or V0 on the first step and for any all-zero column.
// One 256-thread block per column k of the rp padded ones (the leading
// blocks of the residual kernel's grid, so the two run as one launch).  The
// column is read twice (the zero test, then the values, from cache) so that
// these blocks hold no more registers than the residual tiles.
struct VprepArgs {
  const float *vprev;
  int64_t cols;
  int r, rp, first;
  uint64_t seed;
  __nv_bfloat16 *vthi, *vtlo;
  unsigned *amax;
  unsigned *gbar;  // the orthonormalisation kernels' barrier counters (one per sweep)
};
__device__ __forceinline__ void vprep_column(const VprepArgs &V, int k) {
  if (threadIdx.x == 0) {  // this encode's column maxima and barrier counters start from zero
    V.amax[k] = 0u;
    V.amax[V.rp + k] = 0u;
    if (k < 2) V.gbar[k] = 0u;
  }
  int nz = 0;
  if (k < V.r && !V.first)
    for (int64_t j = threadIdx.x; j < V.cols; j += 256) nz |= V.vprev[j * V.r + k] != 0.0f;
  // a column of V_prev that is entirely zero (a dead direction) restarts from V0
  const bool use_prev = __syncthreads_or(nz) != 0;
  for (int64_t j = threadIdx.x; j < V.cols; j += 256) {
    float v = 0.0f;
    if (k < V.r) v = use_prev ? V.vprev[j * V.r + k] : v0_entry(V.seed, j, V.r, k);
    __nv_bfloat16 hi, lo;
    split_bf16(v, hi, lo);
    V.vthi[(int64_t)k * V.cols + j] = hi;
    V.vtlo[(int64_t)k * V.cols + j] = lo;
  }
}

// ---------------------------------------------------------------- residual pass

// D = (a - ahat) + e split in two bf16 terms, row-major ([rows][cols]): the
// K-major A operand of Y = D V and the MN-major A operand of V = D^T Q.  A
// block covers 64 rows x 64 columns (4 per thread per row pass); the grid's
// first rp blocks prepare the warm start instead (vprep_column).  The inputs
// are read once (evict-first loads), so the split, which both products read
// next, is more likely to stay in L2.  The fp32 D is not stored: the
// reconstruction pass recomputes it bit for bit.
template <typename T>
__global__ void __launch_bounds__(256, 8) lr_delta_kernel(const T *a, const float *ahat, const float *err, int ef_explicit,
                                                       int64_t rows, int64_t cols, __nv_bfloat16 *dhi,
                                                       __nv_bfloat16 *dlo, const VprepArgs V) {
  pdl_enter();
  if ((int)blockIdx.x < V.rp) {  // uniform over the block
    vprep_column(V, (int)blockIdx.x);
    return;
  }
  const int tile = (int)blockIdx.x - V.rp, tiles_x = (int)(cols / 64);
  const int64_t r0 = (int64_t)(tile / tiles_x) * 64, c0 = (int64_t)(tile % tiles_x) * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int lr = ty + 16 * i;
    const int64_t off = (r0 + lr) * cols + c0 + 4 * tx;
    float x[4];
    if constexpr (sizeof(T) == 2) {
      const uint2 raw = __ldcs(reinterpret_cast<const uint2 *>(a + off));
      x[0] = __uint_as_float(raw.x << 16);
      x[1] = __uint_as_float(raw.x & 0xffff0000u);
      x[2] = __uint_as_float(raw.y << 16);
      x[3] = __uint_as_float(raw.y & 0xffff0000u);
    } else {
      const float4 f = __ldcs(reinterpret_cast<const float4 *>(a + off));
      x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
    }
    const float4 h = __ldcs(reinterpret_cast<const float4 *>(ahat + off));
    const float4 e = ef_explicit ? __ldcs(reinterpret_cast<const float4 *>(err + off)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float hv[4] = {h.x, h.y, h.z, h.w}, ev[4] = {e.x, e.y, e.z, e.w};
    __nv_bfloat16 hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const float tt = __fsub_rn(x[k], hv[k]);
      const float d = ef_explicit ? __fadd_rn(tt, ev[k]) : tt;
      split_bf16(d, hi[k], lo[k]);
    }
    uint2 ph, pl;
    ph.x = (uint32_t)__bfloat16_as_ushort(hi[0]) | ((uint32_t)__bfloat16_as_ushort(hi[1]) << 16);
    ph.y = (uint32_t)__bfloat16_as_ushort(hi[2]) | ((uint32_t)__bfloat16_as_ushort(hi[3]) << 16);
    pl.x = (uint32_t)__bfloat16_as_ushort(lo[0]) | ((uint32_t)__bfloat16_as_ushort(lo[1]) << 16);
    pl.y = (uint32_t)__bfloat16_as_ushort(lo[2]) | ((uint32_t)__bfloat16_as_ushort(lo[3]) << 16);
    *reinterpret_cast<uint2 *>(dhi + off) = ph;
    *reinterpret_cast<uint2 *>(dlo + off) = pl;
  }
}

// ---------------------------------------------------------------- thin GEMM (tcgen05)

struct ThinArgs {
  float *out;     // [splits][M][n]
  int64_t M;      // rows of A
  int n;          // columns of the product (UMMA N, multiple of 16, <= 128)
  int kblocks;    // K / 64
  int splits;
  int stages;
  int a_mn;       // A stored K x M (M contiguous): loaded in 64 x 64 boxes, MN-major descriptors
  int a_l2;       // L2 priority of A's lines: 0 default, 1 keep (read again later), 2 last use
  int *status;
};

// out[s] = A[:, K_s] * B[:, K_s]^T for the s-th K range, A = ahi + alo
// ([M][K] bf16, K-major; or, with a_mn, [K][M], MN-major), B = bhi + blo
// ([n][K] bf16, K-major), summing the
// products hi*hi + hi*lo + lo*hi in fp32 tensor memory.  One CTA per
// (128-row tile, K split); warp 0 lane 0 streams tiles with TMA into a ring
// of shared-memory stages, warp 1 lane 0 issues the MMAs, all four warps
// read the accumulator back (one row per thread) and write the partial.
__global__ void __launch_bounds__(128, 1)
    lr_thin_gemm_kernel(const __grid_constant__ CUtensorMap ta_hi, const __grid_constant__ CUtensorMap ta_lo,
                        const __grid_constant__ CUtensorMap tb_hi, const __grid_constant__ CUtensorMap tb_lo,
                        const ThinArgs A) {
  pdl_enter();
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ __align__(8) uint64_t full[4], empty[4], accb;
  __shared__ uint32_t tmem_base;
  uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)dsm + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTileM;
  const int s = blockIdx.y;
  const int kb0 = (int)((int64_t)s * A.kblocks / A.splits);
  const int kb1 = (int)((int64_t)(s + 1) * A.kblocks / A.splits);
  const int nk = kb1 - kb0;
  const uint32_t a_bytes = kTileM * kTileK * 2;         // 16 KiB
  const uint32_t b_bytes = (uint32_t)A.n * kTileK * 2;  // n * 128 B (a multiple of 1024 for n % 8 == 0)
  const uint32_t stage_bytes = 2 * a_bytes + 2 * b_bytes;
  const int ST = A.stages;

  if (threadIdx.x == 0) {
    umma::prefetch_tensormap(&ta_hi);
    umma::prefetch_tensormap(&ta_lo);
    umma::prefetch_tensormap(&tb_hi);
    umma::prefetch_tensormap(&tb_lo);
    for (int i = 0; i < ST; i++) {
      umma::mbar_init(&full[i], 1);
      umma::mbar_init(&empty[i], 1);
    }
    umma::mbar_init(&accb, 1);
    umma::fence_barrier_init();
  }
  if (warp == 0) {
    umma::tmem_alloc(&tmem_base, 128);
    umma::tmem_relinquish();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = tmem_base;
  int ok = 1;

  if (warp == 0 && lane == 0) {
    // producer
    const uint64_t pol = A.a_l2 == 1 ? umma::policy_evict_last() : umma::policy_evict_first();
    auto load_a = [&](void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
      if (A.a_l2) umma::tma_load_2d_hint(dst, map, c0, c1, bar, pol);
      else umma::tma_load_2d(dst, map, c0, c1, bar);
    };
    for (int i = 0; i < nk && ok; i++) {
      const int st = i % ST;
      if (i >= ST && !umma::mbar_wait(&empty[st], (uint32_t)(((i / ST) - 1) & 1))) { ok = 0; break; }
      uint8_t *base = sm + (size_t)st * stage_bytes;
      umma::mbar_arrive_expect_tx(&full[st], stage_bytes);
      const int kc = (kb0 + i) * kTileK;
      if (A.a_mn) {  // two 64-column halves of the M tile, 64 K rows each
        load_a(base, &ta_hi, m0, kc, &full[st]);
        load_a(base + a_bytes / 2, &ta_hi, m0 + kTileK, kc, &full[st]);
        load_a(base + a_bytes, &ta_lo, m0, kc, &full[st]);
        load_a(base + a_bytes + a_bytes / 2, &ta_lo, m0 + kTileK, kc, &full[st]);
      } else {
        load_a(base, &ta_hi, kc, m0, &full[st]);
        load_a(base + a_bytes, &ta_lo, kc, m0, &full[st]);
      }
      umma::tma_load_2d(base + 2 * a_bytes, &tb_hi, kc, 0, &full[st]);
      umma::tma_load_2d(base + 2 * a_bytes + b_bytes, &tb_lo, kc, 0, &full[st]);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    const uint32_t idesc = umma::idesc_bf16_f32(kTileM, A.n, A.a_mn != 0);
    for (int i = 0; i < nk && ok; i++) {
      const int st = i % ST;
      if (!umma::mbar_wait(&full[st], (uint32_t)((i / ST) & 1))) { ok = 0; break; }
      umma::fence_after_sync();
      const uint32_t base = umma::saddr(sm + (size_t)st * stage_bytes);
#pragma unroll
      for (int kk = 0; kk < kTileK / 16; kk++) {
        // K-major: the k-th 16-column slice is 32 bytes into each row; MN-major:
        // 16 K rows (2048 bytes) further, the M halves a_bytes / 2 apart
        const uint64_t ah = A.a_mn ? umma::desc_mnmajor_sw128(base + kk * 2048, a_bytes / 2)
                                   : umma::desc_kmajor_sw128(base + kk * 32);
        const uint64_t al = A.a_mn ? umma::desc_mnmajor_sw128(base + a_bytes + kk * 2048, a_bytes / 2)
                                   : umma::desc_kmajor_sw128(base + a_bytes + kk * 32);
        const uint64_t bh = umma::desc_kmajor_sw128(base + 2 * a_bytes + kk * 32);
        const uint64_t bl = umma::desc_kmajor_sw128(base + 2 * a_bytes + b_bytes + kk * 32);
        umma::mma_bf16(tmem, ah, bh, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        umma::mma_bf16(tmem, ah, bl, idesc, 1u);
        umma::mma_bf16(tmem, al, bh, idesc, 1u);
      }
      umma::mma_commit(&empty[st]);
    }
    umma::mma_commit(&accb);
  }
  __syncwarp();
  if (ok) ok = umma::mbar_wait(&accb, 0) ? 1 : 0;
  if (!__syncthreads_and(ok)) {
    if (threadIdx.x == 0) atomicOr(A.status, kStatusTimeout);
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, 128);
    return;
  }
  umma::fence_after_sync();
  // epilogue: thread = accumulator row m0 + 32 warp + lane
  const int64_t row = m0 + 32 * warp + lane;
  float *dst = A.out + ((int64_t)s * A.M + row) * A.n;
  for (int c = 0; c < A.n; c += 16) {
    float v[16];
    umma::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c, v);
    float4 *d4 = reinterpret_cast<float4 *>(dst + c);
    d4[0] = make_float4(v[0], v[1], v[2], v[3]);
    d4[1] = make_float4(v[4], v[5], v[6], v[7]);
    d4[2] = make_float4(v[8], v[9], v[10], v[11]);
    d4[3] = make_float4(v[12], v[13], v[14], v[15]);
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------- CholeskyQR2 pieces

// Rows per partial Gram block (rows are a multiple of 128).
constexpr int kGramRows = 32;

// The fp64 products of the orthonormalisation (the Gram matrices X^T X and
// Q = X M) run on the fp64 tensor-core MMA: tcgen05 has no f64 kind, so this
// is the warp-level mma.sync of shape m8n8k4.  One call adds A B to the 8 x 8
// tile D, A 8 x 4 and B 4 x 8; lane l holds A[l / 4][l % 4], B[l % 4][l / 4]
// and D[l / 4][2 (l % 4)], D[l / 4][2 (l % 4) + 1].  Every result below is
// the same sequence of these calls wherever it is computed, so the kernels
// that fuse two steps give bit-identical values to the separate ones.
__device__ __forceinline__ void dmma_8x8x4(double &d0, double &d1, double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
      : "+d"(d0), "+d"(d1)
      : "d"(a), "d"(b));
}

// Row stride (floats) of a Gram input tile [kGramRows][n]: n + 8 is 8 or 24
// modulo 32, so the 4 rows x 8 columns a fragment load touches fall in 32
// distinct banks.
template <int TT>
__host__ __device__ constexpr int gram_ld() {
  return 16 * TT + 8;
}

// Partial Gram matrix X^T X of the kGramRows rows of xs (fp32 [kGramRows][ld],
// ld = gram_ld) into g (fp64 [n][n], n = 16 TT): the 8 x 8 tiles on and below
// the diagonal (the reduction reads nothing else), dealt round-robin in
// row-major order to the block's 8 warps, each tile the sum over the rows in
// steps of 4 from zero.  The products of two fp32 values are exact in fp64.
template <int TT>
__device__ __forceinline__ void gram_tiles(const float *xs, double *g, int warp, int lane) {
  constexpr int n = 16 * TT, ld = gram_ld<TT>(), CT = 2 * TT, T = CT * (CT + 1) / 2, TPW = (T + 7) / 8;
  const int gq = lane >> 2, t4 = lane & 3;
  int ti[TPW], tj[TPW];
  double acc[TPW][2];
#pragma unroll
  for (int u = 0; u < TPW; u++) {
    int t = warp + 8 * u, I = 0;
    if (t < T) {
      while (t >= I + 1) {
        t -= I + 1;
        I++;
      }
      ti[u] = I;
      tj[u] = t;
    } else {
      ti[u] = -1;
      tj[u] = 0;
    }
    acc[u][0] = acc[u][1] = 0.0;
  }
#pragma unroll
  for (int k0 = 0; k0 < kGramRows; k0 += 4) {
    const float *xr = xs + (k0 + t4) * ld + gq;
#pragma unroll
    for (int u = 0; u < TPW; u++)
      if (ti[u] >= 0) dmma_8x8x4(acc[u][0], acc[u][1], (double)xr[8 * ti[u]], (double)xr[8 * tj[u]]);
  }
#pragma unroll
  for (int u = 0; u < TPW; u++)
    if (ti[u] >= 0)
      *reinterpret_cast<double2 *>(g + (8 * ti[u] + gq) * n + 8 * tj[u] + 2 * t4) = make_double2(acc[u][0], acc[u][1]);
}

// Row block rb (kGramRows rows): X = sum of the nsrc partial slabs of src
// (fixed order), stored fp32 [rows][n], and the partial Gram matrix X^T X
// (fp64, gram_tiles) of these rows into gpart[rb]; tile: kGramRows x gram_ld
// floats of shared memory.  Called by every thread of the block.
template <int TT>
__device__ __forceinline__ void gram_rows(const float *src, int nsrc, int64_t rows, int rb, float *x, double *gpart,
                                          float *tile) {
  constexpr int n = 16 * TT;
  constexpr int n4 = n / 4;                          // float4 per row
  constexpr int NV = (kGramRows * n4 + 255) / 256;   // float4 per thread
  const int64_t r0 = (int64_t)rb * kGramRows;
  const float4 *s4 = reinterpret_cast<const float4 *>(src) + r0 * n4;
  const int64_t slab4 = rows * n4;
  float4 acc4[NV];
  for (int p0 = 0; p0 < nsrc; p0 += 4) {  // four slabs' loads in flight, added in slab order
    float4 t[4][NV];
#pragma unroll
    for (int u = 0; u < 4; u++)
#pragma unroll
      for (int v = 0; v < NV; v++) {
        const int e = threadIdx.x + 256 * v;
        t[u][v] = (p0 + u < nsrc && e < kGramRows * n4) ? __ldcg(s4 + (int64_t)(p0 + u) * slab4 + e)
                                                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
    for (int u = 0; u < 4; u++) {
      if (p0 + u >= nsrc) break;
#pragma unroll
      for (int v = 0; v < NV; v++) {
        if (p0 + u == 0) {
          acc4[v] = t[0][v];
        } else {
          acc4[v].x = __fadd_rn(acc4[v].x, t[u][v].x);
          acc4[v].y = __fadd_rn(acc4[v].y, t[u][v].y);
          acc4[v].z = __fadd_rn(acc4[v].z, t[u][v].z);
          acc4[v].w = __fadd_rn(acc4[v].w, t[u][v].w);
        }
      }
    }
  }
  float4 *x4 = reinterpret_cast<float4 *>(x) + r0 * n4;
  __syncthreads();  // the previous row block's Gram products are done with the tile
#pragma unroll
  for (int v = 0; v < NV; v++) {
    const int e = threadIdx.x + 256 * v;
    if (e < kGramRows * n4) {
      x4[e] = acc4[v];
      const int rr = e / n4, c = (e % n4) * 4;
      *reinterpret_cast<float4 *>(tile + rr * gram_ld<TT>() + c) = acc4[v];
    }
  }
  __syncthreads();
  gram_tiles<TT>(tile, gpart + (int64_t)rb * n * n, threadIdx.x >> 5, threadIdx.x & 31);
}

// Offset of entry (i, j), j <= i, in the Cholesky factor's packed array of
// 8 x 8 tiles (tile (I, J), J <= I, at I (I + 1) / 2 + J; rows of kCholTld
// doubles).
constexpr int kCholTld = 9;  // tile row stride (doubles): a half-warp's 4 x 4 fragment in distinct banks
__host__ __device__ constexpr int chol_tile(int I, int J) { return (I * (I + 1) / 2 + J) * 8 * kCholTld; }
__device__ __forceinline__ int chol_entry(int i, int j) { return chol_tile(i >> 3, j >> 3) + (i & 7) * kCholTld + (j & 7); }

// Entry group g (32 consecutive entries of the n x n matrix, one per lane):
// G = sum over the nblk partial Gram matrices, lower triangle only (the
// Cholesky factor reads nothing above the diagonal; those entries are set to
// zero), row-major into G and, in the Cholesky factor's packed tile layout,
// into Gp (the lower tiles; entries above the diagonal of a diagonal tile are
// zero).  The block's 8 warps sum 8 contiguous slices of the partials (four
// interleaved accumulators, sixteen loads in flight), and the slice sums are
// added in slice order, so the result does not depend on scheduling.  part:
// 8 x 32 doubles of shared memory.  Called by every thread of the block.
__device__ __forceinline__ void reduce_group(const double *gpart, int nblk, int n, double *G, double *Gp, int g,
                                             double (*part)[32]) {
  const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
  const int nn = n * n;
  const int e = g * 32 + lane;
  const bool live = e < nn && (e % n) <= (e / n);
  const int per = (nblk + 7) / 8;
  const int b0 = wp * per, b1 = min(nblk, b0 + per);
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
  if (live) {
    for (int c0 = b0; c0 < b1; c0 += 16) {
      double t[16];
#pragma unroll
      for (int u = 0; u < 16; u++) t[u] = c0 + u < b1 ? __ldcg(gpart + (int64_t)(c0 + u) * nn + e) : 0.0;
      // the partials in order, partial b to accumulator (b - b0) % 4 (b1 - b0 is not always a multiple of 4)
#pragma unroll
      for (int u = 0; u < 16; u += 4) {
        if (c0 + u + 3 < b1) {
          a0 += t[u];
          a1 += t[u + 1];
          a2 += t[u + 2];
          a3 += t[u + 3];
        } else {
#pragma unroll
          for (int w = 0; w < 4; w++)
            if (c0 + u + w < b1) a0 += t[u + w];
        }
      }
    }
  }
  __syncthreads();  // the previous group's slice sums have been read
  part[wp][lane] = (a0 + a1) + (a2 + a3);
  __syncthreads();
  if (wp == 0 && e < nn) {
    double t = part[0][lane];
#pragma unroll
    for (int w = 1; w < 8; w++) t += part[w][lane];
    G[e] = live ? t : 0.0;
    const int gi = e / n, gj = e - (e / n) * n;
    if ((gj >> 3) <= (gi >> 3)) Gp[chol_entry(gi, gj)] = live ? t : 0.0;
  }
}

// ---- Cholesky factor of the Gram matrix and its inverse (fp64)
//
// Blocked right-looking elimination on 8 x 8 tiles.  The working matrix A
// (the lower triangle of G) and X = L^-1 live in shared memory as packed
// lower-triangular arrays of tiles, tile (I, J), J <= I, at index
// I (I + 1) / 2 + J, each 8 rows of chol_tld doubles.  For each block column
// b of the nbl = ceil(nlive / 8) live ones:
//   diagonal  one warp factors the 8 x 8 block A_bb = L_bb L_bb^T column by
//             column in registers (lane i holds row i) and forms X_bb =
//             L_bb^-1 by forward substitution of the identity, row k of it
//             being r_k (e_k - sum_{m<k} L_km X_m) with r_k = 1 / L_kk;
//   panel     L_ib = A_ib X_bb^T for the tiles below, and the finished row
//             of the inverse X_bj = X_bb X_bj (j < b);
//   trailing  A_ij -= L_ib L_jb^T (b < j <= i) and X_ij -= L_ib X_bj
//             (i > b, j <= b).
// The diagonal chain is the critical path, so warp 0 runs one block column
// ahead of the rest: in the step of column b it forms the panel tile
// L_{b+1,b}, applies it to A_{b+1,b+1} and factors that tile, while warps
// 1-7 form the other panel tiles and then (after a named barrier that warp
// 0 arrives at once L_{b+1,b} is stored) the other trailing updates; one
// block barrier ends the step.  Every tile receives the same products in
// the same order as in a plain blocked elimination.  The tile products run
// on the fp64 MMA.  A pivot <= 1e-12 G_00 (R_kk <= 1e-6 R_00), or a column
// at or past nlive (the rank's zero padding), marks column k rank
// deficient: dead[k] = 1, r_k = 0, so row k of X and column k of L (hence
// of X) are zero and the column updates nothing; the other columns are the
// Cholesky factor of G restricted to them.
//
// The factor leaves shared memory as X in the same packed tile layout (all
// chol_ntiles tiles, those past the live ones zero): a flat copy here, and
// the apply phase stages M = X^T from it.

template <int TT>
__host__ __device__ constexpr int chol_ntiles() {
  return (2 * TT) * (2 * TT + 1) / 2;
}
__host__ __device__ constexpr size_t chol_smem_tt(int tt) {
  return (size_t)2 * ((2 * tt) * (2 * tt + 1) / 2) * 8 * kCholTld * 8;
}


// D += sa P R^T (rt) or D += sa P R (!rt) for 8 x 8 tiles P, R of the packed
// arrays, D in this lane's two accumulator entries; sa = -1 subtracts.
__device__ __forceinline__ void chol_tile_mma(double &d0, double &d1, const double *P, const double *R, bool rt,
                                              double sa, int gq, int t4) {
#pragma unroll
  for (int kc = 0; kc < 2; kc++) {
    const double a = sa * P[gq * kCholTld + 4 * kc + t4];
    const double b = rt ? R[gq * kCholTld + 4 * kc + t4] : R[(4 * kc + t4) * kCholTld + gq];
    dmma_8x8x4(d0, d1, a, b);
  }
}

// Factor the diagonal tile of block column b (one warp): reads A_bb, writes
// X_bb = L_bb^-1 and the dead flags of its 8 columns.
__device__ __forceinline__ void chol_diag(const double *Ab, double *Xb, int b, int nlive, double thr, int lane,
                                          int *dead_s) {
  const int i = lane;
  double a[8], y[8], l[8];
#pragma unroll
  for (int j = 0; j < 8; j++) {
    a[j] = (i < 8 && j <= i) ? Ab[i * kCholTld + j] : 0.0;
    y[j] = (i == j) ? 1.0 : 0.0;
  }
  unsigned dmask = 0;
#pragma unroll
  for (int k = 0; k < 8; k++) {
    const double d = __shfl_sync(0xffffffffu, a[k], k);
    const bool dk = 8 * b + k >= nlive || !(d > thr);
    const double r = dk ? 0.0 : rsqrt(d);
    dmask |= dk ? 1u << k : 0u;
    l[k] = i > k ? a[k] * r : 0.0;  // L[i][k]
    // row k of the inverse, then its subtraction from the rows below
    double xk[8];
#pragma unroll
    for (int j = 0; j <= k; j++) xk[j] = __shfl_sync(0xffffffffu, y[j], k) * r;
    if (i == k) {
#pragma unroll
      for (int j = 0; j <= k; j++) y[j] = xk[j];
    }
#pragma unroll
    for (int j = 0; j <= k; j++)
      if (i > k) y[j] = fma(-l[k], xk[j], y[j]);
#pragma unroll
    for (int j = k + 1; j < 8; j++) {
      const double lj = __shfl_sync(0xffffffffu, l[k], j);
      if (i >= j) a[j] = fma(-l[k], lj, a[j]);
    }
  }
  if (i < 8) {
#pragma unroll
    for (int j = 0; j < 8; j++) Xb[i * kCholTld + j] = j <= i ? y[j] : 0.0;
    dead_s[8 * b + i] = (dmask >> i) & 1u;
  }
}

// Named barrier 1 over the whole block: warps 1-7 wait in it, warp 0 only
// arrives (after its shared-memory stores, which the barrier publishes).
__device__ __forceinline__ void chol_bar_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void chol_bar_arrive() { asm volatile("bar.arrive 1, 256;" ::: "memory"); }

// Cholesky factor L of the Gram matrix G (fp64, lower triangle read) and X =
// L^-1 (fp64, packed lower tiles into Xout, as described above), with the
// dead flags.
//
// near_id > 0 (the second pass of CholeskyQR2, where G = Q1^T Q1 is close to
// the identity): if every entry of E = G - I between nonzero columns has
// |E_ij| <= near_id, X is the first-order factor instead: with G = L L^T and
// L = I + F, F = strict_lower(E) + diag(E) / 2 + O(|E|^2), so L^-1 = I - F +
// O(|E|^2), and Q1 X^T has an orthogonality error of about 3 n near_id^2 per
// entry.  A column of G that is exactly zero (a column of Q1 zeroed as rank
// deficient by the first pass) is dead, as in the elimination.  Otherwise
// the blocked elimination runs.
//
// Columns nlive .. n-1 must be zero in G (the padding of the rank).  G
// (row-major, read only by the first-order test) and Xout may alias: G is
// read before the first barrier.
//
// First pass of a sweep (first_pass): the elimination also bounds the
// condition number of X (the matrix being orthonormalised) by B =
// ||L||_F ||L^-1||_F >= kappa_2(L) = kappa_2(X), with ||L||_F^2 the trace of G
// over the live columns, and sets *skip2 when B^2 <= kappa2_max (0: never).
// Then Q1 = X L^-T is orthonormal to within about n kappa^2 2^-53 per entry
// (the fp64 Gram matrix and elimination), far below the fp32 rounding of the
// stored Q (2^-24), and the second pass is skipped.
//
// Run by one block of 256 threads; csm: chol_smem_tt(TT) bytes of shared
// memory (16-byte aligned), dead_s and gdiag: n entries, red: 8.  G and Gp
// were written by other blocks of the same grid: they are read through L2.
template <int TT>
__device__ __forceinline__ void chol_factor(const double *G, const double *Gp, double *Xout, int *dead,
                                            double near_id, int nlive, int *skip2, int first_pass, double kappa2_max,
                                            uint8_t *csm, int *dead_s, double *gdiag, double *red) {
  constexpr int n = 16 * TT;
  constexpr int nall = chol_ntiles<TT>() * 8 * kCholTld;  // doubles of the whole packed array
  if (near_id > 0.0) {
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    const int i0 = ty * TT, j0 = tx * TT;
    const bool lower = tx <= ty;  // blocks above the diagonal hold nothing
    double w[TT][TT];
#pragma unroll
    for (int a = 0; a < TT; a++)
#pragma unroll
      for (int c = 0; c < TT; c++) w[a][c] = (lower && j0 + c <= i0 + a) ? __ldcg(G + (i0 + a) * n + j0 + c) : 0.0;
    int far = 0;
    if (lower) {
#pragma unroll
      for (int a = 0; a < TT; a++)
#pragma unroll
        for (int c = 0; c < TT; c++) {
          const int gi = i0 + a, gj = j0 + c;
          const double g = w[a][c];
          if (gj < gi ? !(fabs(g) <= near_id) : (gj == gi && g != 0.0 && !(fabs(g - 1.0) <= near_id))) far = 1;
        }
    }
    if (!__syncthreads_or(far)) {
      // first-order factor; zero diagonal entries mark dead columns
      if (tx == ty) {
#pragma unroll
        for (int a = 0; a < TT; a++) dead_s[i0 + a] = w[a][a] == 0.0 ? 1 : 0;
      }
      __syncthreads();
      // every entry of the packed tiles (the part above the diagonal of a
      // diagonal tile is zero); the tiles' padding column is never read
#pragma unroll
      for (int a = 0; a < TT; a++) {
        const int gi = i0 + a;
#pragma unroll
        for (int c = 0; c < TT; c++) {
          const int gj = j0 + c;
          if ((gj >> 3) > (gi >> 3)) continue;
          double m = 0.0;  // X[gi][gj] = L^-1[gi][gj]
          if (lower && gj <= gi && !dead_s[gi] && !dead_s[gj]) m = gj == gi ? 1.0 - 0.5 * (w[a][c] - 1.0) : -w[a][c];
          Xout[chol_entry(gi, gj)] = m;
        }
      }
      for (int e = threadIdx.x; e < n; e += blockDim.x) dead[e] = dead_s[e];
      return;
    }
  }
  double *A = reinterpret_cast<double *>(csm);  // packed tiles of the working matrix
  double *X = A + chol_ntiles<TT>() * 8 * kCholTld;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, t4 = lane & 3;
  const int nbl = (min(max(nlive, 0), n) + 7) / 8;
  const int nl = 8 * nbl;
  // the working matrix: the live tiles of G's packed copy (the first
  // nbl (nbl + 1) / 2 tiles of both arrays), sixteen loads in flight per thread
  const int nlt = nbl * (nbl + 1) / 2 * 8 * kCholTld;
  for (int e0 = 0; e0 < nlt; e0 += 16 * 256) {
    double g[16];
#pragma unroll
    for (int u = 0; u < 16; u++) {
      const int e = e0 + u * 256 + (int)threadIdx.x;
      g[u] = e < nlt ? __ldcg(Gp + e) : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 16; u++) {
      const int e = e0 + u * 256 + (int)threadIdx.x;
      if (e < nlt) {
        A[e] = g[u];
        X[e] = 0.0;
      }
    }
  }
  for (int k = nl + threadIdx.x; k < n; k += blockDim.x) dead_s[k] = 1;
  __syncthreads();
  // G's diagonal (for the condition bound), read before any update of A
  for (int k = threadIdx.x; k < nl; k += blockDim.x) gdiag[k] = A[chol_entry(k, k)];
  const double thr = 1e-12 * A[0];
  if (nbl > 0 && warp == 0) chol_diag(A, X, 0, nlive, thr, lane, dead_s);
  __syncthreads();
  for (int b = 0; b < nbl; b++) {
    const int m = nbl - 1 - b;  // block rows below the diagonal
    const double *Xbb = X + chol_tile(b, b);
    if (warp == 0) {
      if (m > 0) {  // uniform: the next diagonal tile's chain
        double *P = A + chol_tile(b + 1, b);
        double p0 = 0.0, p1 = 0.0;
        chol_tile_mma(p0, p1, P, Xbb, true, 1.0, gq, t4);
        __syncwarp();
        P[gq * kCholTld + 2 * t4] = p0;
        P[gq * kCholTld + 2 * t4 + 1] = p1;
        __syncwarp();
        chol_bar_arrive();  // L_{b+1,b} is stored: warps 1-7 may start the trailing updates
        double *T = A + chol_tile(b + 1, b + 1);
        double d0 = T[gq * kCholTld + 2 * t4], d1 = T[gq * kCholTld + 2 * t4 + 1];
        chol_tile_mma(d0, d1, P, P, true, -1.0, gq, t4);
        T[gq * kCholTld + 2 * t4] = d0;
        T[gq * kCholTld + 2 * t4 + 1] = d1;
        __syncwarp();
        chol_diag(T, X + chol_tile(b + 1, b + 1), b + 1, nlive, thr, lane, dead_s);
      }
    } else {
      // panel L_ib = A_ib X_bb^T (i >= b + 2) and the inverse's row X_bj = X_bb X_bj (j < b)
      const int mp = m > 0 ? m - 1 : 0;
      for (int t = warp - 1; t < mp + b; t += 7) {
        double *T = t < mp ? A + chol_tile(b + 2 + t, b) : X + chol_tile(b, t - mp);
        double d0 = 0.0, d1 = 0.0;
        if (t < mp)
          chol_tile_mma(d0, d1, T, Xbb, true, 1.0, gq, t4);
        else
          chol_tile_mma(d0, d1, Xbb, T, false, 1.0, gq, t4);
        __syncwarp();
        T[gq * kCholTld + 2 * t4] = d0;
        T[gq * kCholTld + 2 * t4 + 1] = d1;
      }
      if (m > 0) {  // uniform
        chol_bar_sync();  // every panel tile of column b is stored
        // trailing A_ij -= L_ib L_jb^T (b < j <= i, all but the next diagonal tile) and X_ij -= L_ib X_bj
        // (i > b, j <= b)
        const int ntr = m * (m + 1) / 2, ntask = ntr - 1 + m * (b + 1);
        for (int t = warp - 1; t < ntask; t += 7) {
          int i, j;
          double *T;
          const double *R;
          bool rt;
          if (t < ntr - 1) {  // trailing tile, row-major over the triangle after the next diagonal tile
            int u = t + 1, ii = 0;
            while (u >= ii + 1) {
              u -= ii + 1;
              ii++;
            }
            i = b + 1 + ii;
            j = b + 1 + u;
            T = A + chol_tile(i, j);
            R = A + chol_tile(j, b);
            rt = true;
          } else {
            const int u = t - (ntr - 1);
            i = b + 1 + u / (b + 1);
            j = u % (b + 1);
            T = X + chol_tile(i, j);
            R = X + chol_tile(b, j);
            rt = false;
          }
          double d0 = T[gq * kCholTld + 2 * t4], d1 = T[gq * kCholTld + 2 * t4 + 1];
          chol_tile_mma(d0, d1, A + chol_tile(i, b), R, rt, -1.0, gq, t4);
          T[gq * kCholTld + 2 * t4] = d0;
          T[gq * kCholTld + 2 * t4 + 1] = d1;
        }
      }
    }
    __syncthreads();
  }
  // X to Xout, the whole packed array (tiles past the live ones zero)
  double sx = 0.0;  // this thread's part of ||X||_F^2 (the padding column and the zeros add nothing)
  for (int e = threadIdx.x; e < nall; e += blockDim.x) {
    const double xv = e < nlt ? X[e] : 0.0;
    Xout[e] = xv;
    sx = fma(xv, xv, sx);
  }
  for (int e = threadIdx.x; e < n; e += blockDim.x) dead[e] = dead_s[e];
  if (first_pass) {  // uniform over the block
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
    if (lane == 0) red[warp] = sx;
    __syncthreads();
    if (warp == 0) {
      double tr = 0.0;  // trace of G over the live columns
      for (int k = lane; k < nl; k += 32)
        if (!dead_s[k]) tr += gdiag[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tr += __shfl_xor_sync(0xffffffffu, tr, o);
      if (lane == 0) {
        double xs2 = 0.0;
        for (int w = 0; w < 8; w++) xs2 += red[w];
        *skip2 = (kappa2_max > 0.0 && tr * xs2 <= kappa2_max) ? 1 : 0;
      }
    }
  }
}

// The second CholeskyQR pass of a sweep is skipped when the first pass bounds
// the condition number of the matrix it orthonormalises by this (see
// chol_factor): its orthogonality error is then about n kSkipKappa^2 2^-53
// <= 2^-30 per entry for n <= 128, against the 2^-24 of the stored fp32 Q.
constexpr double kSkipKappa = 256.0;
template <int TT>
__host__ __device__ constexpr int apply_xld() {
  return 16 * TT + 4;  // X tile row stride (floats): 4 or 20 mod 32, a fragment's 8 rows x 4 in distinct banks
}
template <int TT>
__host__ __device__ constexpr int apply_mld() {
  return 16 * TT + 4;  // M row stride (doubles): each half-warp's 4 rows x 4 fragment entries in distinct banks
}

// Stage M = L^-T into Ms (row stride apply_mld) from the Cholesky factor's
// packed tiles of X = L^-1 (tile (I, J) of X is the transpose of M's tile
// (J, I); the entries of M below its diagonal tiles are never read), and
// with it the kGramRows rows of X from row r0 (apply_stage_x), all loads in
// flight at once.  Xp was written by another block of the grid: it is read
// through L2.
template <int TT>
__device__ __forceinline__ void apply_stage_mx(const double *Xp, double *Ms, const float *x, int64_t rows, int64_t r0,
                                               float *xs) {
  constexpr int n = 16 * TT, mld = apply_mld<TT>(), xld = apply_xld<TT>();
  constexpr int NT = chol_ntiles<TT>(), NE = NT * 64, NU = (NE + 255) / 256;
  constexpr int NX = kGramRows * n / 4, NXU = (NX + 255) / 256;
  double v[NU];
  float4 xv[NXU];
#pragma unroll
  for (int u = 0; u < NU; u++) {  // all loads in flight first
    const int e = (int)threadIdx.x + 256 * u;
    const int t = e >> 6, w = e & 63;
    v[u] = e < NE ? __ldcg(Xp + t * 8 * kCholTld + (w & 7) * kCholTld + (w >> 3)) : 0.0;
  }
  const float4 *x4 = reinterpret_cast<const float4 *>(x) + r0 * (n / 4);
#pragma unroll
  for (int u = 0; u < NXU; u++) {
    const int e = (int)threadIdx.x + 256 * u;
    xv[u] = (e < NX && r0 + e / (n / 4) < rows) ? x4[e] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < NXU; u++) {
    const int e = (int)threadIdx.x + 256 * u;
    if (e < NX) *reinterpret_cast<float4 *>(xs + (e / (n / 4)) * xld + (e % (n / 4)) * 4) = xv[u];
  }
#pragma unroll
  for (int u = 0; u < NU; u++) {
    const int e = (int)threadIdx.x + 256 * u;
    if (e < NE) {
      const int t = e >> 6, w = e & 63;
      int I = 0, J = t;  // t = I (I + 1) / 2 + J, J <= I
      while (J > I) {
        J -= I + 1;
        I++;
      }
      Ms[(8 * J + (w >> 3)) * mld + 8 * I + (w & 7)] = v[u];
    }
  }
}

// Stage the nx rows of X (fp32 [rows][n]) from row r0 into xs (row stride
// apply_xld); rows past the end read as zero.
template <int TT>
__device__ __forceinline__ void apply_stage_x(const float *x, int64_t rows, int64_t r0, int nx, float *xs) {
  constexpr int n = 16 * TT, xld = apply_xld<TT>();
  const float4 *x4 = reinterpret_cast<const float4 *>(x) + r0 * (n / 4);
  for (int e = threadIdx.x; e < nx * n / 4; e += blockDim.x) {
    const int rr = e / (n / 4), c = (e % (n / 4)) * 4;
    const float4 val = r0 + rr < rows ? x4[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4 *>(xs + rr * xld + c) = val;
  }
}

// Column tile (of 8) that warp w computes in its round jt of Q = X M: the
// 2 TT tiles are dealt in descending order (the widest term ranges first),
// snake-wise over the 8 warps; -1 past the last.
template <int TT>
__device__ __forceinline__ int apply_ctile(int w, int jt) {
  const int s = 8 * jt + ((jt & 1) ? 7 - w : w);
  return s < 2 * TT ? 2 * TT - 1 - s : -1;
}
template <int TT>
__host__ __device__ constexpr int apply_rounds() {
  return (2 * TT + 7) / 8;
}

// Q = X M for the 8 RT rows of xs (M upper triangular): warp w computes its
// column tiles (apply_ctile) for all RT row tiles, each output the sum from
// zero over M's rows 0 .. 8 J + 7 in steps of 4 (the rows below add zeros).
template <int TT, int RT>
__device__ __forceinline__ void apply_tiles(const float *xs, const double *Ms, int warp, int lane,
                                            double (&acc)[apply_rounds<TT>()][RT][2]) {
  constexpr int mld = apply_mld<TT>(), xld = apply_xld<TT>();
  const int gq = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int jt = 0; jt < apply_rounds<TT>(); jt++) {
#pragma unroll
    for (int i = 0; i < RT; i++) acc[jt][i][0] = acc[jt][i][1] = 0.0;
    const int J = apply_ctile<TT>(warp, jt);
    if (J < 0) continue;  // uniform over the warp
    const double *mp = Ms + t4 * mld + 8 * J + gq;
    const float *xp = xs + gq * xld + t4;
#pragma unroll 2
    for (int k0 = 0; k0 < 8 * J + 8; k0 += 4) {
      const double b = mp[k0 * mld];
#pragma unroll
      for (int i = 0; i < RT; i++) dmma_8x8x4(acc[jt][i][0], acc[jt][i][1], (double)xp[8 * i * xld + k0], b);
    }
  }
}

// The outputs of Q = X M for the 8 RT rows of one block from r0, from the
// accumulators of apply_tiles: Q fp32 [rows][n]; when amax != nullptr the
// absmax of each of Q's first r columns (the INT4 scales' input), one
// atomicMax per column and block (cmax: n entries of shared memory, zeroed
// before the block's last barrier); when qthi != nullptr Q^T split in bf16
// ([n][rows], the K-major B operand of V = D^T Q), transposed through qs
// (shared, n x (8 RT + 1) floats, free once every thread has passed the
// first barrier here) so that those stores are row-contiguous.  Every thread
// of the block calls this (amax and qthi are uniform).
template <int TT, int RT>
__device__ __forceinline__ void apply_store(const double (&acc)[apply_rounds<TT>()][RT][2], int64_t r0, int64_t rows,
                                            float *q, __nv_bfloat16 *qthi, __nv_bfloat16 *qtlo, int r,
                                            unsigned *amax, unsigned *cmax, float *qs, int warp, int lane) {
  constexpr int n = 16 * TT, NR = 8 * RT, qld = NR + 1, JR = apply_rounds<TT>();
  const int gq = lane >> 2, t4 = lane & 3;
  float res[JR][RT][2];
#pragma unroll
  for (int jt = 0; jt < JR; jt++) {
    const int J = apply_ctile<TT>(warp, jt);
    uint32_t m0 = 0u, m1 = 0u;  // this lane's column maxima over its rows (bit patterns of |Q| >= 0)
#pragma unroll
    for (int i = 0; i < RT; i++) {
      res[jt][i][0] = (float)acc[jt][i][0];
      res[jt][i][1] = (float)acc[jt][i][1];
      const int64_t row = r0 + 8 * i + gq;
      if (J >= 0 && row < rows) {
        const int c = 8 * J + 2 * t4;
        *reinterpret_cast<float2 *>(q + row * n + c) = make_float2(res[jt][i][0], res[jt][i][1]);
        m0 = max(m0, __float_as_uint(fabsf(res[jt][i][0])));
        m1 = max(m1, __float_as_uint(fabsf(res[jt][i][1])));
      }
    }
    if (amax != nullptr && J >= 0) {  // uniform over the warp: the INT4 column maxima of Q
      // the 8 lanes of a column pair (lane bits 2-4) first, then one shared atomic per column and warp
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        m0 = max(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = max(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      }
      if (gq == 0) {
        const int c = 8 * J + 2 * t4;
        atomicMax(&cmax[c], m0);
        atomicMax(&cmax[c + 1], m1);
      }
    }
  }
  __syncthreads();  // the column maxima are complete, and every thread is done with the buffer under qs
  if (amax != nullptr) {  // uniform over the block
    for (int c = threadIdx.x; c < r; c += 256)
      if (cmax[c]) atomicMax(&amax[c], cmax[c]);
  }
  if (qthi == nullptr) return;  // uniform over the block
#pragma unroll
  for (int jt = 0; jt < JR; jt++) {
    const int J = apply_ctile<TT>(warp, jt);
    if (J < 0) continue;
#pragma unroll
    for (int i = 0; i < RT; i++) {
      const int c = 8 * J + 2 * t4;
      qs[c * qld + 8 * i + gq] = res[jt][i][0];
      qs[(c + 1) * qld + 8 * i + gq] = res[jt][i][1];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n * NR; e += 256) {
    const int c = e / NR, rr = e % NR;
    if (r0 + rr < rows) {
      __nv_bfloat16 hi, lo;
      split_bf16(qs[c * qld + rr], hi, lo);
      qthi[(int64_t)c * rows + r0 + rr] = hi;
      qtlo[(int64_t)c * rows + r0 + rr] = lo;
    }
  }
}

// Q = X M (M = L^-T, upper triangular, zero below the diagonal; staged once
// from the packed factor Xp) for the grid's row blocks of kGramRows rows
// (apply_tiles; the rows of X staged in shared memory).  final_q: the
// outputs of apply_store (Q, its INT4 column maxima when amax != nullptr,
// Q^T split when qthi != nullptr); otherwise (the first pass of a sweep
// whose second pass runs) Q and the partial Gram matrix Q^T Q of each row
// block from the fp32 values it stores, with the sums of gram_tiles, into
// gpart.  x and q may alias (a block reads its rows before it writes them).
// sm: apply_gram_smem(n) bytes of shared memory; cmax: n entries.  Called by
// every thread of the block.
template <int TT>
__device__ __forceinline__ void apply_phase(const float *x, const double *Xp, int64_t rows, int nblk, float *q,
                                            double *gpart, bool final_q, __nv_bfloat16 *qthi, __nv_bfloat16 *qtlo,
                                            int r, unsigned *amax, uint8_t *sm, unsigned *cmax) {
  constexpr int n = 16 * TT, mld = apply_mld<TT>(), xld = apply_xld<TT>(), RT = kGramRows / 8;
  constexpr int JR = apply_rounds<TT>();
  static_assert(kGramRows * xld >= n * (kGramRows + 1), "the X tile holds the transposed Q tile");
  double *Ms = reinterpret_cast<double *>(sm);          // [n][mld]
  float *xs = reinterpret_cast<float *>(Ms + n * mld);  // [kGramRows][xld]
  float *gs = xs + kGramRows * xld;                     // Q1 [kGramRows][gram_ld]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, t4 = lane & 3;
  if ((int)blockIdx.x >= nblk) return;  // uniform: no row block here
  apply_stage_mx<TT>(Xp, Ms, x, rows, (int64_t)blockIdx.x * kGramRows, xs);
  if (final_q && amax != nullptr)
    for (int c = threadIdx.x; c < n; c += 256) cmax[c] = 0u;
  for (int rb = blockIdx.x; rb < nblk; rb += gridDim.x) {
    const int64_t r0 = (int64_t)rb * kGramRows;
    if (rb != (int)blockIdx.x) {
      __syncthreads();  // the previous row block is done with xs and gs
      apply_stage_x<TT>(x, rows, r0, kGramRows, xs);
    }
    __syncthreads();
    double acc[JR][RT][2];
    apply_tiles<TT, RT>(xs, Ms, warp, lane, acc);
    if (final_q) {
      apply_store<TT, RT>(acc, r0, rows, q, qthi, qtlo, r, amax, cmax, xs, warp, lane);
      continue;
    }
#pragma unroll
    for (int jt = 0; jt < JR; jt++) {
      const int J = apply_ctile<TT>(warp, jt);
      if (J < 0) continue;
#pragma unroll
      for (int i = 0; i < RT; i++) {
        const int64_t row = r0 + 8 * i + gq;
        const int c = 8 * J + 2 * t4;
        const float2 v = row < rows ? make_float2((float)acc[jt][i][0], (float)acc[jt][i][1]) : make_float2(0.f, 0.f);
        if (row < rows) *reinterpret_cast<float2 *>(q + row * n + c) = v;
        *reinterpret_cast<float2 *>(gs + (8 * i + gq) * gram_ld<TT>() + c) = v;
      }
    }
    __syncthreads();
    gram_tiles<TT>(gs, gpart + (int64_t)rb * n * n, warp, lane);
  }
}

// ---- the orthonormalisation of one sweep as one persistent kernel
//
// CholeskyQR2 of the split-K partials of Y: the first pass (Gram matrix of X
// = their sum, Cholesky factor, Q1 = X L^-T) and, unless the first pass
// bounds kappa(X) by kSkipKappa, the second (the same on Q1).  Its phases
// are separated by grid-wide barriers instead of kernel boundaries: the
// Gram rows (every block), the reduction of the partial Gram matrices (every
// block), the factor (block 0), the apply (every block), and so on.  All
// blocks must be resident at once: the grid is at most the SMs times the
// blocks that fit on one (checked on the host), and each barrier gives up
// after spin_limit polls, reporting a timeout in *status.

struct OrthoArgs {
  const float *src;    // the split-K partials of Y [nsrc][rows][n]
  int nsrc;
  int64_t rows;
  int nblk;            // row blocks of kGramRows rows
  float *x;            // X = the sum of the partials [rows][n]
  float *q;            // Q [rows][n]
  double *gpart;       // partial Gram matrices [nblk][n][n]
  double *L;           // reduced Gram matrix (row-major), then the packed factor L^-1
  double *Gp;          // the reduced Gram matrix in packed tiles
  int *dead, *skip2;
  int nlive;           // the rank (columns nlive .. n-1 are padding)
  double near_id;      // the second pass's first-order bound (lr_qr2_tol)
  double kappa2_max;   // the skip test's bound on kappa^2 (0: never skip)
  __nv_bfloat16 *qthi, *qtlo;
  int r;
  unsigned *amax;      // the INT4 column maxima of Q (nullptr: not the last sweep)
  unsigned *gbar;      // this sweep's barrier counter, zero at launch
  int *status;
  uint32_t spin_limit;
  int withhold_arrival;  // test hook: block 0 does not arrive at the first barrier, so every block's wait runs out
};

template <int TT>
struct OrthoShared {
  int dead_s[16 * TT];
  double gdiag[16 * TT];
  double red[8];
  double part[8][32];
  unsigned cmax[16 * TT];
  int ok;
};

// Grid-wide barrier number k (1, 2, ...) of the launch: every block adds one
// to the counter and waits until it reaches k gridDim.x.  The block's writes
// are ordered before its arrival by the block barrier and the release of the
// add, and the other blocks' writes before everything after the wait by the
// acquiring poll and the block barrier after it; data written by other blocks
// is still read through L2 (ld.cg).  False (uniform over the block, after
// the status is set) when the wait ran out.
__device__ __forceinline__ bool ortho_sync(const OrthoArgs &A, unsigned k, int *ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!(A.withhold_arrival && k == 1 && blockIdx.x == 0))
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(A.gbar) : "memory");
    const unsigned target = k * gridDim.x;
    int good = 0;
    for (uint32_t it = 0; it < A.spin_limit; it++) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(A.gbar) : "memory");
      if (v >= target) {
        good = 1;
        break;
      }
    }
    if (!good) atomicOr(A.status, kStatusTimeout);
    *ok = good;
  }
  __syncthreads();
  return *ok != 0;
}

template <int TT>
__global__ void __launch_bounds__(256, 1) lr_ortho_kernel(const OrthoArgs A) {
  pdl_enter();
  constexpr int n = 16 * TT;
  extern __shared__ __align__(16) uint8_t osm[];
  __shared__ OrthoShared<TT> sh;
  const int ngroups = (n * n + 31) / 32;
  unsigned nb = 0;
  // first pass: the Gram rows of X = sum of the partials
  for (int rb = blockIdx.x; rb < A.nblk; rb += gridDim.x)
    gram_rows<TT>(A.src, A.nsrc, A.rows, rb, A.x, A.gpart, reinterpret_cast<float *>(osm));
  if (!ortho_sync(A, ++nb, &sh.ok)) return;
  for (int g = blockIdx.x; g < ngroups; g += gridDim.x) reduce_group(A.gpart, A.nblk, n, A.L, A.Gp, g, sh.part);
  if (!ortho_sync(A, ++nb, &sh.ok)) return;
  if (blockIdx.x == 0)
    chol_factor<TT>(A.L, A.Gp, A.L, A.dead, 0.0, A.nlive, A.skip2, 1, A.kappa2_max, osm, sh.dead_s, sh.gdiag, sh.red);
  if (!ortho_sync(A, ++nb, &sh.ok)) return;
  const bool final_q = __ldcg(A.skip2) != 0;  // uniform over the grid
  apply_phase<TT>(A.x, A.L, A.rows, A.nblk, A.q, A.gpart, final_q, A.qthi, A.qtlo, A.r, A.amax, osm, sh.cmax);
  if (final_q) return;
  // second pass on Q1
  if (!ortho_sync(A, ++nb, &sh.ok)) return;
  for (int g = blockIdx.x; g < ngroups; g += gridDim.x) reduce_group(A.gpart, A.nblk, n, A.L, A.Gp, g, sh.part);
  if (!ortho_sync(A, ++nb, &sh.ok)) return;
  if (blockIdx.x == 0)
    chol_factor<TT>(A.L, A.Gp, A.L, A.dead, A.near_id, A.nlive, A.skip2, 0, 0.0, osm, sh.dead_s, sh.gdiag, sh.red);
  if (!ortho_sync(A, ++nb, &sh.ok)) return;
  apply_phase<TT>(A.q, A.L, A.rows, A.nblk, A.q, nullptr, true, A.qthi, A.qtlo, A.r, A.amax, osm, sh.cmax);
}

// V = sum of the partial slabs (fixed order) [cols][n]; V_prev (state,
// [cols][r]) = V[:, :r]; when vthi != nullptr also V^T split for the next
// iteration's Y = D V; when amax != nullptr the absmax of each of V's first r
// columns (the INT4 scales' input) goes to amax, one atomicMax per column
// and block.
__global__ void __launch_bounds__(256) lr_vsum_kernel(const float *vpart, int nsrc, int64_t cols, int n, int r,
                                                      float *v, float *vprev, __nv_bfloat16 *vthi,
                                                      __nv_bfloat16 *vtlo, unsigned *amax) {
  pdl_enter();
  __shared__ unsigned cmax[kMaxRank];  // n <= kMaxRank
  if (amax != nullptr) {  // uniform over the grid
    for (int c = threadIdx.x; c < n; c += blockDim.x) cmax[c] = 0u;
    __syncthreads();
  }
  const int64_t total = cols * n;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.0f;
    for (int p0 = 0; p0 < nsrc; p0 += 8) {  // eight slabs' loads in flight, added in slab order
      float t[8];
#pragma unroll
      for (int u = 0; u < 8; u++) t[u] = p0 + u < nsrc ? vpart[(int64_t)(p0 + u) * total + idx] : 0.0f;
#pragma unroll
      for (int u = 0; u < 8; u++)
        if (p0 + u < nsrc) acc = p0 + u == 0 ? t[0] : __fadd_rn(acc, t[u]);
    }
    const uint32_t j = (uint32_t)idx / (uint32_t)n;
    const int k = (int)((uint32_t)idx - j * (uint32_t)n);
    v[idx] = acc;
    if (k < r) vprev[j * r + k] = acc;
    if (amax != nullptr) atomicMax(&cmax[k], __float_as_uint(fabsf(acc)));
    if (vthi) {
      __nv_bfloat16 hi, lo;
      split_bf16(k < r ? acc : 0.0f, hi, lo);
      vthi[(int64_t)k * cols + j] = hi;
      vtlo[(int64_t)k * cols + j] = lo;
    }
  }
  if (amax != nullptr) {  // the block's column maxima, one atomicMax per column
    __syncthreads();
    for (int c = threadIdx.x; c < r; c += blockDim.x)
      if (cmax[c]) atomicMax(&amax[c], cmax[c]);
  }
}

// ---------------------------------------------------------------- INT4 payload

struct PackArgs {
  uint8_t *payload;  // header + body
  const float *q;    // [rows][n]
  const float *v;    // [cols][n]
  int64_t rows, cols;
  int r, n, int4;
  int64_t sec1, sec2, body;
  Header hdr;
  unsigned *amax;  // [2 n]: column absmax bit patterns of Q, then of V (zeroed by vprep_column)
  // the sender's reconstruction operands, written from the packed values (the
  // dequantisation of the payload, see lr_dequant_kernel); k >= r stays zero
  int kp;
  __nv_bfloat16 *uahi, *ualo, *vbhi, *vblo;
};

// Scale s_k = fp32(absmax_k / 7) of column k of U (k < r) or V (k >= r).
__device__ __forceinline__ float lr_scale_of(const PackArgs &P, int k) {
  const unsigned bits = k < P.r ? P.amax[k] : P.amax[P.n + k - P.r];
  return (float)((double)__uint_as_float(bits) / 7.0);
}

__device__ __forceinline__ uint32_t int4_code(float x, float s) {
  if (s == 0.0f) return 0;
  double t = rint((double)x / (double)s);
  t = t > 7.0 ? 7.0 : (t < -7.0 ? -7.0 : t);
  return (uint32_t)((int)t & 0xF);
}

// Reconstruction operand entry (i, k) of U (isv false) or of the scaled V
// from the value the payload carries: INT4, the code q (U: q, exact in bf16;
// V: fp32(q sU_k sV_k), products in fp64); fp32 factors, the value itself.
__device__ __forceinline__ void lr_operand_store(__nv_bfloat16 *hi_out, __nv_bfloat16 *lo_out, int64_t o, float x) {
  __nv_bfloat16 hi, lo;
  split_bf16(x, hi, lo);
  hi_out[o] = hi;
  if (lo_out) lo_out[o] = lo;
}

// Nibbles of U and V (element (i,k) is nibble i*r + k, low nibble first) or
// the fp32 factors, padding bytes zero, and the header; and the sender's
// reconstruction operands from the same values, exactly as the dequantisation
// of the payload computes them.
__global__ void __launch_bounds__(256) lr_pack_kernel(PackArgs P) {
  pdl_enter();
  uint8_t *body = P.payload + kHdrBytes;
  if (blockIdx.x == 0 && threadIdx.x < 16) reinterpret_cast<uint32_t *>(P.payload)[threadIdx.x] = P.hdr.w[threadIdx.x];
  const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (P.int4) {
    // the scale section: block 0 writes the 2r scales, every thread computes
    // the ones it needs the same way
    float *sc = reinterpret_cast<float *>(body);
    if (blockIdx.x == 0)
      for (int k = threadIdx.x; k < 2 * P.r; k += blockDim.x) sc[k] = lr_scale_of(P, k);
    // scale section padding
    for (int64_t b = (int64_t)P.r * 8 + tid; b < P.sec1; b += nthr) body[b] = 0;
    const uint32_t ubytes = (uint32_t)(P.sec2 - P.sec1), vbytes = (uint32_t)(P.body - P.sec2);
    const uint32_t un = (uint32_t)(P.rows * P.r), vn = (uint32_t)(P.cols * P.r), r = (uint32_t)P.r;
    for (uint32_t b = (uint32_t)tid; b < ubytes + vbytes; b += (uint32_t)nthr) {
      const bool isv = b >= ubytes;
      const uint32_t bb = isv ? b - ubytes : b;
      const uint32_t nel = isv ? vn : un;
      const float *m = isv ? P.v : P.q;
      uint32_t byte = 0;
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const uint32_t e = 2 * bb + h;
        if (e < nel) {
          const uint32_t i = e / r, k = e - i * r;
          const uint32_t c = int4_code(m[(int64_t)i * P.n + k], lr_scale_of(P, (int)k + (isv ? P.r : 0)));
          byte |= c << (4 * h);
          const int q = (c & 0x8) ? (int)c - 16 : (int)c;
          const int64_t o = (int64_t)i * P.kp + k;
          if (isv)
            lr_operand_store(P.vbhi, P.vblo, o,
                             (float)((double)q * (double)lr_scale_of(P, (int)k) * (double)lr_scale_of(P, P.r + (int)k)));
          else
            lr_operand_store(P.uahi, nullptr, o, (float)q);
        }
      }
      body[(isv ? P.sec2 : P.sec1) + bb] = (uint8_t)byte;
    }
  } else {
    float *u = reinterpret_cast<float *>(body);
    float *vv = reinterpret_cast<float *>(body + P.sec2);
    const int64_t un = P.rows * P.r, vn = P.cols * P.r;
    for (int64_t e = tid; e < un; e += nthr) {
      const int64_t i = e / P.r, k = e % P.r;
      const float x = P.q[i * P.n + k];
      u[e] = x;
      lr_operand_store(P.uahi, P.ualo, i * P.kp + k, x);
    }
    for (int64_t e = tid; e < vn; e += nthr) {
      const int64_t i = e / P.r, k = e % P.r;
      const float x = P.v[i * P.n + k];
      vv[e] = x;
      lr_operand_store(P.vbhi, P.vblo, i * P.kp + k, x);
    }
    for (int64_t b = un * 4 + tid; b < P.sec2; b += nthr) body[b] = 0;
    for (int64_t b = P.sec2 + vn * 4 + tid; b < P.body; b += nthr) body[b] = 0;
  }
}

__device__ __forceinline__ int nibble_at(const uint8_t *base, int64_t idx) {
  const int v = (idx & 1) ? (base[idx >> 1] >> 4) : (base[idx >> 1] & 0xF);
  return (v & 0x8) ? v - 16 : v;
}

// Reconstruction operands from the payload alone (the receiver; the sender's
// pack kernel writes the same values): A = U
// ([rows][kp]; INT4: the integer codes, exact in bf16; fp32 factors: split),
// B = V scaled ([cols][kp], split; INT4: fp32(qV * sU * sV) per entry).
struct DequantArgs {
  const uint8_t *payload;
  int64_t rows, cols;
  int r, kp, int4;
  int64_t sec1, sec2;
  __nv_bfloat16 *uahi, *ualo, *vbhi, *vblo;
  int check_header;
  Header expect;
  int *status;
};

__global__ void __launch_bounds__(256) lr_dequant_kernel(DequantArgs D) {
  pdl_enter();
  if (D.check_header && !lr_header_ok(D.payload, D.expect, D.status)) return;
  const uint8_t *body = D.payload + kHdrBytes;
  const float *sc = reinterpret_cast<const float *>(body);
  // one warp per row: rows of U first, then rows of V; lanes over the kp columns
  const int lane = threadIdx.x & 31;
  const int64_t nwarp = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = D.rows + D.cols;
  for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < total; row += nwarp) {
    const bool isv = row >= D.rows;
    const int64_t i = isv ? row - D.rows : row;
    const uint8_t *nb = body + (isv ? D.sec2 : D.sec1);
    const float *f = reinterpret_cast<const float *>(body + (isv ? D.sec2 : 0));
    for (int k = lane; k < D.kp; k += 32) {
      float x = 0.0f;
      if (k < D.r) {
        if (D.int4) {
          const int q = nibble_at(nb, i * D.r + k);
          x = isv ? (float)((double)q * (double)sc[k] * (double)sc[D.r + k]) : (float)q;
        } else {
          x = f[i * D.r + k];
        }
      }
      __nv_bfloat16 hi, lo;
      split_bf16(x, hi, lo);
      const int64_t o = i * D.kp + k;
      if (isv) {
        D.vbhi[o] = hi;
        D.vblo[o] = lo;
      } else {
        D.uahi[o] = hi;
        if (D.ualo) D.ualo[o] = lo;
      }
    }
  }
}

// ---------------------------------------------------------------- reconstruction GEMM (tcgen05)

struct ReconArgs {
  int64_t rows, cols;
  int kblocks;        // kp / 64
  int a_split;        // 1: A carries a lo term (fp32 factors)
  int ef_explicit;
  int ef_off;  // CF_EF_OFF: ahat <- fp32(a), e untouched
  const void *a;      // sender: activations [rows][cols]
  float *ahat;
  float *err;
  void *recon;        // receiver
  int *status;
  const uint8_t *payload;
  int check_header;
  Header expect;
  uint32_t spin_limit;  // polls of the operand wait
  int withhold_copies;  // test hook: issue no operand copy, so that wait runs out
};

// C tile (128 rows x 128 cols) = A[rows tile] * B[cols tile]^T over K = kp,
// products hi*hi + hi*lo (+ lo*hi when A is split), then the fused update:
// sender: D = (a - ahat) + e recomputed bit for bit; e = D - C; ahat = ahat + C;
// receiver: ahat = ahat + C; recon = cast(ahat).
// 8 warps: warp 0 lane 0 loads the operands (TMA) and issues the MMAs; after
// they complete, warp w drains TMEM lanes 32 (w % 4).., columns 64 (w / 4)..
// into a padded shared-memory C tile (the operand buffers are free by then),
// and all warps update whole rows with coalesced 512-byte accesses, in
// batches of rows whose HBM operands are loaded together (the first batch
// before the MMAs).  The role is a template parameter so that the receiver,
// which loads only the state, takes larger batches.
constexpr int kReconThreads = 256;
constexpr int kCsLd = kReconN + 4;  // padded C-tile row (floats)
constexpr int kReconBatchSender = 4;  // rows per warp and batch of the update
constexpr int kReconBatchReceiver = 8;

// The update's global operands for one batch of a warp's rows (lane l:
// columns 4l .. 4l + 3): the state, and for the sender the error (explicit
// feedback) and the activation.
template <typename T, bool SENDER>
struct ReconRows {
  static constexpr int B = SENDER ? kReconBatchSender : kReconBatchReceiver;
  static constexpr int NB = kTileM / (8 * B);
  static_assert(NB * 8 * B == kTileM, "update batches must cover the tile");
  using X = typename std::conditional<sizeof(T) == 2, uint2, float4>::type;
  float4 h[B];
  float4 e[SENDER ? B : 1];
  X x[SENDER ? B : 1];  // the activation as loaded
  __device__ __forceinline__ void load(const ReconArgs &R, int64_t m0, int64_t n0, int warp, int lane, int b) {
#pragma unroll
    for (int u = 0; u < B; u++) {
      const int rr = warp + 8 * (B * b + u);
      const int64_t off = (m0 + rr) * R.cols + n0 + 4 * lane;
      h[u] = __ldcs(reinterpret_cast<const float4 *>(R.ahat + off));
      if constexpr (SENDER) {
        e[u] = R.ef_explicit ? __ldcs(reinterpret_cast<const float4 *>(R.err + off)) : make_float4(0.f, 0.f, 0.f, 0.f);
        x[u] = __ldcs(reinterpret_cast<const X *>(static_cast<const T *>(R.a) + off));
      }
    }
  }
  __device__ __forceinline__ void act(int u, float (&v)[4]) const {
    if constexpr (sizeof(T) == 2) {
      v[0] = __uint_as_float(x[u].x << 16);
      v[1] = __uint_as_float(x[u].x & 0xffff0000u);
      v[2] = __uint_as_float(x[u].y << 16);
      v[3] = __uint_as_float(x[u].y & 0xffff0000u);
    } else {
      v[0] = x[u].x; v[1] = x[u].y; v[2] = x[u].z; v[3] = x[u].w;
    }
  }
};

template <typename T, bool SENDER>
__global__ void __launch_bounds__(kReconThreads, 2)
    lr_recon_kernel(const __grid_constant__ CUtensorMap ta_hi, const __grid_constant__ CUtensorMap ta_lo,
                    const __grid_constant__ CUtensorMap tb_hi, const __grid_constant__ CUtensorMap tb_lo,
                    const ReconArgs R) {
  pdl_enter();
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ __align__(8) uint64_t full, accb;
  __shared__ uint32_t tmem_base;
  if (R.check_header && !lr_header_ok(R.payload, R.expect, R.status)) return;
  uint8_t *sm = reinterpret_cast<uint8_t *>(((uintptr_t)dsm + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kTileM, n0 = (int64_t)blockIdx.y * kReconN;
  const uint32_t tile = kTileM * kTileK * 2;  // 16 KiB per 128 x 64 tile
  const int nkb = R.kblocks;
  // layout: A hi [nkb] | A lo [nkb] (if split) | B hi [nkb] | B lo [nkb]
  const uint32_t off_al = nkb * tile;
  const uint32_t off_bh = off_al + (R.a_split ? nkb * tile : 0);
  const uint32_t off_bl = off_bh + nkb * tile;
  const uint32_t total = off_bl + nkb * tile;

  if (threadIdx.x == 0) {
    umma::mbar_init(&full, 1);
    umma::mbar_init(&accb, 1);
    umma::fence_barrier_init();
  }
  if (warp == 0) {
    umma::tmem_alloc(&tmem_base, 128);
    umma::tmem_relinquish();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = tmem_base;
  ReconRows<T, SENDER> L;
  L.load(R, m0, n0, warp, lane, 0);
  {
    // the rows of the later update batches go to L2 meanwhile (a bulk
    // prefetch holds no register): lane l < (NB - 1) B of warp w takes row
    // w + 8 (B b + u) of the tile, b = 1 + l / B, u = l % B
    constexpr int Bq = ReconRows<T, SENDER>::B, NBq = ReconRows<T, SENDER>::NB;
    if (lane < (NBq - 1) * Bq) {
      const int rr = warp + 8 * (Bq * (1 + lane / Bq) + lane % Bq);
      const int64_t off = (m0 + rr) * R.cols + n0;
      umma::prefetch_l2(R.ahat + off, kReconN * 4);
      if constexpr (SENDER) {
        if (R.ef_explicit) umma::prefetch_l2(R.err + off, kReconN * 4);
        umma::prefetch_l2(static_cast<const T *>(R.a) + off, kReconN * (uint32_t)sizeof(T));
      }
    }
  }
  int ok = 1;
  if (warp == 0 && lane == 0) {
    umma::mbar_arrive_expect_tx(&full, total);
    // (with the test hook no copy is issued: the barrier's transaction count
    // stays pending, the wait below gives up, and nothing is left in flight)
    for (int kb = 0; kb < nkb && !R.withhold_copies; kb++) {
      umma::tma_load_2d(sm + kb * tile, &ta_hi, kb * kTileK, (int)m0, &full);
      if (R.a_split) umma::tma_load_2d(sm + off_al + kb * tile, &ta_lo, kb * kTileK, (int)m0, &full);
      umma::tma_load_2d(sm + off_bh + kb * tile, &tb_hi, kb * kTileK, (int)n0, &full);
      umma::tma_load_2d(sm + off_bl + kb * tile, &tb_lo, kb * kTileK, (int)n0, &full);
    }
    if (!umma::mbar_wait(&full, 0, R.spin_limit)) {
      ok = 0;
    } else {
      umma::fence_after_sync();
      const uint32_t idesc = umma::idesc_bf16_f32(kTileM, kReconN);
      const uint32_t base = umma::saddr(sm);
      for (int kb = 0; kb < nkb; kb++) {
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; kk++) {
          const uint32_t o = kb * tile + kk * 32;
          const uint64_t ah = umma::desc_kmajor_sw128(base + o);
          const uint64_t bh = umma::desc_kmajor_sw128(base + off_bh + o);
          const uint64_t bl = umma::desc_kmajor_sw128(base + off_bl + o);
          umma::mma_bf16(tmem, ah, bh, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma::mma_bf16(tmem, ah, bl, idesc, 1u);
          if (R.a_split) umma::mma_bf16(tmem, umma::desc_kmajor_sw128(base + off_al + o), bh, idesc, 1u);
        }
      }
      umma::mma_commit(&accb);
    }
  }
  __syncwarp();
  if (!__syncthreads_and(ok)) {
    if (threadIdx.x == 0) atomicOr(R.status, kStatusTimeout);
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, 128);
    return;
  }
  ok = umma::mbar_wait(&accb, 0) ? 1 : 0;
  if (!__syncthreads_and(ok)) {
    if (threadIdx.x == 0) atomicOr(R.status, kStatusTimeout);
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, 128);
    return;
  }
  umma::fence_after_sync();
  // TMEM -> shared C tile (the MMAs are complete: the operand buffers are free)
  float *cs = reinterpret_cast<float *>(sm);
  {
    const int q = warp & 3, hf = warp >> 2;
    float *dst = cs + (32 * q + lane) * kCsLd + hf * 64;
#pragma unroll
    for (int c = 0; c < 64; c += 16) {
      float v[16];
      umma::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(hf * 64 + c), v);
      float4 *d4 = reinterpret_cast<float4 *>(dst + c);
      d4[0] = make_float4(v[0], v[1], v[2], v[3]);
      d4[1] = make_float4(v[4], v[5], v[6], v[7]);
      d4[2] = make_float4(v[8], v[9], v[10], v[11]);
      d4[3] = make_float4(v[12], v[13], v[14], v[15]);
    }
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, 128);
  // coalesced update: warp w takes rows w + 8 j; lane l columns 4l .. 4l + 3;
  // batch b = rows j in [B b, B (b + 1))
  constexpr int B = ReconRows<T, SENDER>::B;
  for (int b = 0; b < ReconRows<T, SENDER>::NB; b++) {
    if (b > 0) L.load(R, m0, n0, warp, lane, b);
#pragma unroll
    for (int u = 0; u < B; u++) {
      const int rr = warp + 8 * (B * b + u);
      const int64_t off = (m0 + rr) * R.cols + n0 + 4 * lane;
      const float4 cv = *reinterpret_cast<const float4 *>(cs + rr * kCsLd + 4 * lane);
      const float c[4] = {cv.x, cv.y, cv.z, cv.w};
      const float h[4] = {L.h[u].x, L.h[u].y, L.h[u].z, L.h[u].w};
      float hn[4];
#pragma unroll
      for (int k = 0; k < 4; k++) hn[k] = __fadd_rn(h[k], c[k]);
      if constexpr (SENDER) {
        float xv[4];
        L.act(u, xv);
        if (R.ef_off) {  // no error feedback: the state is the activation
          __stcs(reinterpret_cast<float4 *>(R.ahat + off), make_float4(xv[0], xv[1], xv[2], xv[3]));
          continue;
        }
        __stcs(reinterpret_cast<float4 *>(R.ahat + off), make_float4(hn[0], hn[1], hn[2], hn[3]));
        const float e[4] = {L.e[u].x, L.e[u].y, L.e[u].z, L.e[u].w};
        float en[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const float tt = __fsub_rn(xv[k], h[k]);
          const float d = R.ef_explicit ? __fadd_rn(tt, e[k]) : tt;
          en[k] = __fsub_rn(d, c[k]);
        }
        __stcs(reinterpret_cast<float4 *>(R.err + off), make_float4(en[0], en[1], en[2], en[3]));
      } else {
        __stcs(reinterpret_cast<float4 *>(R.ahat + off), make_float4(hn[0], hn[1], hn[2], hn[3]));
        if constexpr (sizeof(T) == 2) {
          uint2 w;
          w.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hn[0])) |
                ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hn[1])) << 16);
          w.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hn[2])) |
                ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hn[3])) << 16);
          __stcs(reinterpret_cast<uint2 *>(static_cast<T *>(R.recon) + off), w);
        } else {
          __stcs(reinterpret_cast<float4 *>(static_cast<T *>(R.recon) + off), make_float4(hn[0], hn[1], hn[2], hn[3]));
        }
      }
    }
  }
}

// ---------------------------------------------------------------- host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    (void)cudaGetLastError();
  }
  return fn;
}

// bf16 [outer][inner] row-major, box {64, box_rows}, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)kTileK, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Bytes of G in the Cholesky factor's packed layout: the lower 8 x 8 tiles of
// an rp x rp matrix, rows of kCholTld doubles.
size_t gpk_bytes(size_t rp) { return (rp / 8) * (rp / 8 + 1) / 2 * 8 * kCholTld * 8; }

size_t thin_smem(int n, int stages) { return (size_t)stages * (2u * kTileM * kTileK * 2 + 2u * n * kTileK * 2) + 1024; }
int thin_stages(int n) { return n <= 96 ? 4 : 3; }
size_t recon_smem(int kblocks, int a_split) {
  const size_t ops = (size_t)kblocks * kTileM * kTileK * 2 * (3 + a_split);
  const size_t ctile = (size_t)kTileM * kCsLd * 4;
  return (ops > ctile ? ops : ctile) + 1024;
}
cudaError_t set_recon_smem(int smem) {
  const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(lr_recon_kernel<__nv_bfloat16, true>, attr, smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(lr_recon_kernel<__nv_bfloat16, false>, attr, smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(lr_recon_kernel<float, true>, attr, smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(lr_recon_kernel<float, false>, attr, smem)) != cudaSuccess)
    return e;
  return cudaSuccess;
}
// The dynamic shared-memory limit is one setting per kernel and device,
// shared by every low-rank state (and the allocation-free decode).  The
// kernels whose request depends on the rank -- the thin GEMM and the
// reconstruction -- therefore get the largest request of any supported rank,
// so that setting up a state of one rank never lowers the limit below what a
// live state of another rank launches with.  The value is the same on every
// call, so concurrent set-ups agree.
cudaError_t set_shared_smem_limits() {
  size_t thin = 0;
  for (int n = 16; n <= kMaxRank; n += 16) {
    const size_t b = thin_smem(n, thin_stages(n));
    if (b > thin) thin = b;
  }
  const cudaError_t e =
      cudaFuncSetAttribute(lr_thin_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)thin);
  if (e != cudaSuccess) return e;
  return set_recon_smem((int)recon_smem(kMaxRank / kTileK, 1));
}
size_t apply_gram_smem(int n) {  // n = 16 TT: apply_mld = apply_xld = n + 4, gram_ld = n + 8
  return (size_t)n * (n + 4) * 8 + (size_t)kGramRows * (n + 4) * 4 + (size_t)kGramRows * (n + 8) * 4;
}
// Dynamic shared memory of the orthonormalisation kernel: its phases use the
// same buffer (the Gram tile, the Cholesky tiles, the apply operands).
size_t ortho_smem(int n) {
  const size_t a = apply_gram_smem(n), c = chol_smem_tt(n / 16), g = (size_t)kGramRows * (n + 8) * 4;
  return a > c ? (a > g ? a : g) : (c > g ? c : g);
}
// Polls of a grid barrier of the orthonormalisation kernel before it gives up.
constexpr uint32_t kOrthoSpinLimit = 1u << 20;

}  // namespace

void lowrank_plan(int64_t rows, int64_t cols, const cf_params &p, LowrankPlan *plan) {
  plan->rows = rows;
  plan->cols = cols;
  plan->rank = p.rank;
  plan->iters = p.iters;
  plan->int4 = p.lr_int4;
  plan->batch = p.batch;
  plan->role = p.role;
  plan->dtype = p.dtype;
  plan->ef_explicit = p.ef == CF_EF_EXPLICIT;
  plan->ef_off = p.ef == CF_EF_OFF;
  plan->qr2_tol = p.lr_qr2_tol;
  plan->rp = round_up(p.rank < 16 ? 16 : p.rank, 16);
  plan->kp = round_up(p.rank, kTileK);
  plan->supported = rows % 128 == 0 && cols % 128 == 0 && rows >= 128 && cols >= 128 && p.batch == 1 &&
                    p.rank >= 1 && p.rank <= 128 && rows < (1ll << 30) && cols < (1ll << 30) &&
                    (rows + cols) * (int64_t)round_up(p.rank, kTileK) < (1ll << 31);  // 32-bit factor indices
  // split-K so that each thin GEMM fills the SMs: (tiles of 128 rows) x splits
  const int ty = (int)(rows / kTileM), tv = (int)(cols / kTileM);
  const int kby = (int)(cols / kTileK), kbv = (int)(rows / kTileK);
  // one CTA per SM (the operand ring takes most of the shared memory): the
  // largest split count that keeps tiles x splits within one wave
  int nsm = 148, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) !=
                                               cudaSuccess || nsm < 1) {
    (void)cudaGetLastError();
    nsm = 148;
  }
  auto splits = [nsm](int tiles, int kblocks) {
    int s = nsm / tiles;
    if (s > kblocks) s = kblocks;
    return s < 1 ? 1 : s;
  };
  plan->sy = splits(ty, kby);
  plan->sv = splits(tv, kbv);
  const int64_t mx = rows > cols ? rows : cols;
  plan->nblk_gram = (int)(mx / kGramRows);
  const size_t R = (size_t)rows, C = (size_t)cols, rp = (size_t)plan->rp, kp = (size_t)plan->kp;
  size_t dec = 0;
  dec += pad256(R * kp * 2) * 2;  // uahi, ualo
  dec += pad256(C * kp * 2) * 2;  // vbhi, vblo
  size_t enc = dec;
  enc += pad256(R * C * 2) * 2;                               // dhi dlo
  enc += pad256(rp * C * 2) * 2 + pad256(rp * R * 2) * 2;     // vt, qt
  enc += pad256((size_t)plan->sy * R * rp * 4);               // ypart
  enc += pad256((size_t)plan->sv * C * rp * 4);               // vpart
  enc += pad256(mx * rp * 4) * 2 + pad256(C * rp * 4);        // xbuf, q, v
  enc += pad256((size_t)plan->nblk_gram * rp * rp * 8);       // gpart
  enc += pad256(rp * rp * 8) + pad256(rp * 4) + pad256(4);    // L, dead, skip flag
  enc += pad256(2 * 4);                                       // barrier counters of the two sweeps
  enc += pad256(gpk_bytes(rp));                                // G in packed tiles
  enc += pad256(2 * rp * 4);                                  // amax
  plan->enc_scratch_bytes = enc;
  plan->dec_scratch_bytes = dec;
}

namespace {

// The orthonormalisation kernel's shared-memory limit (one value per TT, so
// states of different ranks do not interfere) and the largest grid whose
// blocks are all resident at once.
template <int TT>
cudaError_t set_ortho_tt(int *resident) {
  const int sm = (int)ortho_smem(16 * TT);
  cudaError_t e = cudaFuncSetAttribute(lr_ortho_kernel<TT>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  int occ = 0, nsm = 0, dev = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, lr_ortho_kernel<TT>, 256, sm)) != cudaSuccess) return e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  *resident = occ * nsm;
  return occ > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

cudaError_t set_ortho(int n, int *resident) {
  switch (n / 16) {
    case 1: return set_ortho_tt<1>(resident);
    case 2: return set_ortho_tt<2>(resident);
    case 3: return set_ortho_tt<3>(resident);
    case 4: return set_ortho_tt<4>(resident);
    case 5: return set_ortho_tt<5>(resident);
    case 6: return set_ortho_tt<6>(resident);
    case 7: return set_ortho_tt<7>(resident);
    case 8: return set_ortho_tt<8>(resident);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int lowrank_bind(LowrankPlan *plan, void *scratch) {
  uint8_t *p = static_cast<uint8_t *>(scratch);
  const size_t R = (size_t)plan->rows, C = (size_t)plan->cols, rp = (size_t)plan->rp, kp = (size_t)plan->kp;
  const size_t mx = R > C ? R : C;
  auto take = [&](size_t bytes) {
    uint8_t *q = p;
    p += pad256(bytes);
    return q;
  };
  LowrankBufs &b = plan->b;
  b.uahi = reinterpret_cast<__nv_bfloat16 *>(take(R * kp * 2));
  b.ualo = reinterpret_cast<__nv_bfloat16 *>(take(R * kp * 2));
  b.vbhi = reinterpret_cast<__nv_bfloat16 *>(take(C * kp * 2));
  b.vblo = reinterpret_cast<__nv_bfloat16 *>(take(C * kp * 2));
  bool ok = make_map(&plan->tm_uahi, b.uahi, kp, R, kTileM) && make_map(&plan->tm_ualo, b.ualo, kp, R, kTileM) &&
            make_map(&plan->tm_vbhi, b.vbhi, kp, C, kReconN) && make_map(&plan->tm_vblo, b.vblo, kp, C, kReconN);
  if (plan->role == CF_SENDER) {
    b.dhi = reinterpret_cast<__nv_bfloat16 *>(take(R * C * 2));
    b.dlo = reinterpret_cast<__nv_bfloat16 *>(take(R * C * 2));
    b.vthi = reinterpret_cast<__nv_bfloat16 *>(take(rp * C * 2));
    b.vtlo = reinterpret_cast<__nv_bfloat16 *>(take(rp * C * 2));
    b.qthi = reinterpret_cast<__nv_bfloat16 *>(take(rp * R * 2));
    b.qtlo = reinterpret_cast<__nv_bfloat16 *>(take(rp * R * 2));
    b.ypart = reinterpret_cast<float *>(take((size_t)plan->sy * R * rp * 4));
    b.vpart = reinterpret_cast<float *>(take((size_t)plan->sv * C * rp * 4));
    b.xbuf = reinterpret_cast<float *>(take(mx * rp * 4));
    b.q = reinterpret_cast<float *>(take(mx * rp * 4));
    b.v = reinterpret_cast<float *>(take(C * rp * 4));
    b.gpart = reinterpret_cast<double *>(take((size_t)plan->nblk_gram * rp * rp * 8));
    b.L = reinterpret_cast<double *>(take(rp * rp * 8));
    b.dead = reinterpret_cast<int *>(take(rp * 4));
    b.skip2 = reinterpret_cast<int *>(take(4));
    b.gbar = reinterpret_cast<unsigned *>(take(2 * 4));
    b.gpk = reinterpret_cast<double *>(take(gpk_bytes(rp)));
    b.amax = reinterpret_cast<unsigned *>(take(2 * rp * 4));
    ok = ok && make_map(&plan->tm_dhi, b.dhi, C, R, kTileM) && make_map(&plan->tm_dlo, b.dlo, C, R, kTileM) &&
         make_map(&plan->tm_vthi, b.vthi, C, rp, (uint32_t)rp) && make_map(&plan->tm_vtlo, b.vtlo, C, rp, (uint32_t)rp) &&
         make_map(&plan->tm_dmhi, b.dhi, C, R, kTileK) && make_map(&plan->tm_dmlo, b.dlo, C, R, kTileK) &&
         make_map(&plan->tm_qthi, b.qthi, R, rp, (uint32_t)rp) && make_map(&plan->tm_qtlo, b.qtlo, R, rp, (uint32_t)rp);
  }
  if (!ok) return CF_ERR_CUDA;
  // kernels that need more than 48 KiB of dynamic shared memory
  int resident = 0;
  if (set_shared_smem_limits() != cudaSuccess || set_ortho(plan->rp, &resident) != cudaSuccess) {
    (void)cudaGetLastError();
    return CF_ERR_CUDA;
  }
  const int nblk = (int)(plan->rows / kGramRows);
  plan->ortho_grid = nblk < resident ? nblk : resident;
  return CF_OK;
}

namespace {

cudaError_t launch_thin(const LowrankPlan &P, const CUtensorMap &ah, const CUtensorMap &al, const CUtensorMap &bh,
                        const CUtensorMap &bl, float *out, int64_t M, int64_t K, int splits, int *status,
                        cudaStream_t st, bool a_mn = false, int a_l2 = 0) {
  ThinArgs A{};
  A.out = out;
  A.M = M;
  A.n = P.rp;
  A.kblocks = (int)(K / kTileK);
  A.splits = splits;
  A.stages = thin_stages(P.rp);
  A.a_mn = a_mn ? 1 : 0;
  A.a_l2 = a_l2;
  A.status = status;
  launch_pdl(lr_thin_gemm_kernel, dim3(dim3((unsigned)(M / kTileM), (unsigned)splits)), dim3(128), thin_smem(P.rp, A.stages), st, 
      ah, al, bh, bl, A);
  return cudaGetLastError();
}

// One sweep's CholeskyQR2 of Y (its split-K partials src) into Q: one
// launch of the persistent orthonormalisation kernel, whose first pass
// decides whether the second one runs (lr_qr2_tol = 0: always, the full
// CholeskyQR2).
cudaError_t orthonormalise(const LowrankPlan &P, const float *src, int nsrc, int sweep, unsigned *amax, int *status,
                           cudaStream_t st) {
  const LowrankBufs &b = P.b;
  OrthoArgs A{};
  A.src = src;
  A.nsrc = nsrc;
  A.rows = P.rows;
  A.nblk = (int)(P.rows / kGramRows);
  A.x = b.xbuf;
  A.q = b.q;
  A.gpart = b.gpart;
  A.L = b.L;
  A.Gp = b.gpk;
  A.dead = b.dead;
  A.skip2 = b.skip2;
  A.nlive = P.rank;
  A.near_id = P.qr2_tol;
  A.kappa2_max = P.qr2_tol > 0.0 ? kSkipKappa * kSkipKappa : 0.0;
  A.qthi = b.qthi;
  A.qtlo = b.qtlo;
  A.r = P.rank;
  A.amax = amax;
  A.gbar = b.gbar + sweep;
  A.status = status;
  A.spin_limit = P.test_wait_polls ? P.test_wait_polls : kOrthoSpinLimit;
  A.withhold_arrival = P.test_wait_polls != 0;
  const dim3 grid((unsigned)P.ortho_grid);
  const size_t sm = ortho_smem(P.rp);
  switch (P.rp / 16) {
    case 1: launch_pdl_coop(lr_ortho_kernel<1>, grid, dim3(256), sm, st, A); break;
    case 2: launch_pdl_coop(lr_ortho_kernel<2>, grid, dim3(256), sm, st, A); break;
    case 3: launch_pdl_coop(lr_ortho_kernel<3>, grid, dim3(256), sm, st, A); break;
    case 4: launch_pdl_coop(lr_ortho_kernel<4>, grid, dim3(256), sm, st, A); break;
    case 5: launch_pdl_coop(lr_ortho_kernel<5>, grid, dim3(256), sm, st, A); break;
    case 6: launch_pdl_coop(lr_ortho_kernel<6>, grid, dim3(256), sm, st, A); break;
    case 7: launch_pdl_coop(lr_ortho_kernel<7>, grid, dim3(256), sm, st, A); break;
    case 8: launch_pdl_coop(lr_ortho_kernel<8>, grid, dim3(256), sm, st, A); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

PackArgs pack_args(const LowrankPlan &P, uint8_t *payload, const Header &hdr) {
  PackArgs A{};
  A.payload = payload;
  A.q = P.b.q;
  A.v = P.b.v;
  A.rows = P.rows;
  A.cols = P.cols;
  A.r = P.rank;
  A.n = P.rp;
  A.int4 = P.int4;
  const size_t R = (size_t)P.rows, C = (size_t)P.cols, r = (size_t)P.rank;
  if (P.int4) {
    A.sec1 = (int64_t)pad16(r * 8);
    A.sec2 = A.sec1 + (int64_t)pad16((R * r + 1) / 2);
    A.body = A.sec2 + (int64_t)pad16((C * r + 1) / 2);
  } else {
    A.sec1 = 0;
    A.sec2 = (int64_t)pad16(R * r * 4);
    A.body = A.sec2 + (int64_t)pad16(C * r * 4);
  }
  A.hdr = hdr;
  A.amax = P.b.amax;
  A.kp = P.kp;
  A.uahi = P.b.uahi;
  A.ualo = P.int4 ? nullptr : P.b.ualo;
  A.vbhi = P.b.vbhi;
  A.vblo = P.b.vblo;
  return A;
}

cudaError_t dequant_and_recon(const LowrankPlan &P, const uint8_t *payload, bool receiver, const Header &expect,
                              const void *a, float *ahat, float *err, void *recon, int *status, cudaStream_t st) {
  const PackArgs pa = pack_args(P, nullptr, expect);
  DequantArgs D{};
  D.payload = payload;
  D.rows = P.rows;
  D.cols = P.cols;
  D.r = P.rank;
  D.kp = P.kp;
  D.int4 = P.int4;
  D.sec1 = pa.sec1;
  D.sec2 = pa.sec2;
  D.uahi = P.b.uahi;
  D.ualo = P.int4 ? nullptr : P.b.ualo;
  D.vbhi = P.b.vbhi;
  D.vblo = P.b.vblo;
  D.check_header = receiver;
  D.expect = expect;
  D.status = status;
  // the sender's operands were written by the pack kernel from the same values
  if (receiver) launch_pdl(lr_dequant_kernel, dim3(1184), dim3(256), 0, st, D);
  ReconArgs R{};
  R.rows = P.rows;
  R.cols = P.cols;
  R.kblocks = P.kp / kTileK;
  R.a_split = P.int4 ? 0 : 1;
  R.ef_explicit = P.ef_explicit;
  R.ef_off = P.ef_off;
  R.a = a;
  R.ahat = ahat;
  R.err = err;
  R.recon = recon;
  R.status = status;
  R.payload = payload;
  R.check_header = receiver;
  R.expect = expect;
  R.spin_limit = P.test_wait_polls ? P.test_wait_polls : umma::kSpinLimit;
  R.withhold_copies = P.test_wait_polls != 0;
  const dim3 grid((unsigned)(P.rows / kTileM), (unsigned)(P.cols / kReconN));
  const size_t smem = recon_smem(R.kblocks, R.a_split);
  auto *kern = P.dtype == CF_BF16 ? (receiver ? lr_recon_kernel<__nv_bfloat16, false> : lr_recon_kernel<__nv_bfloat16, true>)
                                  : (receiver ? lr_recon_kernel<float, false> : lr_recon_kernel<float, true>);
  launch_pdl(kern, dim3(grid), dim3(kReconThreads), smem, st, P.tm_uahi, P.tm_ualo, P.tm_vbhi, P.tm_vblo, R);
  return cudaGetLastError();
}

}  // namespace

cudaError_t lowrank_encode(const LowrankPlan &P, const EncArgs &args, const PtrTable *tab, float *vprev,
                           uint64_t step, uint64_t seed, cudaStream_t st) {
  if (tab) return cudaErrorNotSupported;  // batch 1 only
  const LowrankBufs &b = P.b;
  const int64_t R = P.rows, C = P.cols;
  VprepArgs V{};
  V.vprev = vprev;
  V.cols = C;
  V.r = P.rank;
  V.rp = P.rp;
  V.first = step == 1 ? 1 : 0;
  V.seed = seed;
  V.vthi = b.vthi;
  V.vtlo = b.vtlo;
  V.amax = b.amax;
  V.gbar = b.gbar;
  const dim3 dg((unsigned)(P.rp + (C / 64) * (R / 64)));
  if (P.dtype == CF_BF16)
    launch_pdl(lr_delta_kernel<__nv_bfloat16>, dim3(dg), dim3(256), 0, st, static_cast<const __nv_bfloat16 *>(args.a),
               args.ahat, args.err, P.ef_explicit, R, C, b.dhi, b.dlo, V);
  else
    launch_pdl(lr_delta_kernel<float>, dim3(dg), dim3(256), 0, st, static_cast<const float *>(args.a), args.ahat, args.err,
               P.ef_explicit, R, C, b.dhi, b.dlo, V);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  for (int it = 0; it < P.iters; it++) {
    // Y = D V
    if ((e = launch_thin(P, P.tm_dhi, P.tm_dlo, P.tm_vthi, P.tm_vtlo, b.ypart, R, C, P.sy, args.status, st, false,
                         1)) !=
        cudaSuccess)
      return e;
    // the last sweep's Q and V feed the INT4 scales: their column maxima are
    // taken where they are written
    const bool more = it + 1 < P.iters;
    unsigned *amax_q = (P.int4 && !more) ? b.amax : nullptr;
    unsigned *amax_v = (P.int4 && !more) ? b.amax + P.rp : nullptr;
    // Q = orth(Y): CholeskyQR2
    if ((e = orthonormalise(P, b.ypart, P.sy, it, amax_q, args.status, st)) != cudaSuccess) return e;
    // V = D^T Q
    if ((e = launch_thin(P, P.tm_dmhi, P.tm_dmlo, P.tm_qthi, P.tm_qtlo, b.vpart, C, R, P.sv, args.status, st, true,
                         2)) !=
        cudaSuccess)
      return e;
    launch_pdl(lr_vsum_kernel, dim3(592), dim3(256), 0, st, b.vpart, P.sv, C, P.rp, P.rank, b.v, vprev, more ? b.vthi : nullptr,
                                        more ? b.vtlo : nullptr, amax_v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // INT4 (or fp32) factors into the payload
  const PackArgs pa = pack_args(P, args.payload, args.hdr);
  launch_pdl(lr_pack_kernel, dim3(592), dim3(256), 0, st, pa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // sender reconstruction from the payload bytes
  return dequant_and_recon(P, args.payload, false, args.hdr, args.a, args.ahat, args.err, nullptr, args.status, st);
}

cudaError_t lowrank_decode(const LowrankPlan &P, const DecArgs &args, const PtrTable *tab, cudaStream_t st) {
  if (tab) return cudaErrorNotSupported;
  return dequant_and_recon(P, args.payload, true, args.expect, nullptr, args.ahat, nullptr, args.recon, args.status,
                           st);
}

}  // namespace cfi

// ---------------------------------------------------------------- allocation-free decode

namespace cfi {
namespace {

// Fixed scratch of cf_lowrank_decode_noalloc: the dequantised reconstruction
// operands.  Host code must not use the symbol as an address: the device
// address comes from cudaGetSymbolAddress, once per device.
constexpr size_t kNoAllocBytes = 8u << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch for the current device (set-up on first use).
int noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return CF_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      (void)cudaGetLastError();
      return CF_ERR_CUDA;
    }
    if (set_shared_smem_limits() != cudaSuccess) {
      (void)cudaGetLastError();
      return CF_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return CF_OK;
}

}  // namespace
}  // namespace cfi

extern "C" int cf_lowrank_decode_noalloc(int64_t rows, int64_t cols, const cf_params *p, uint64_t step,
                                         const void *payload, float *ahat, void *recon, int *status, void *stream) {
  using namespace cfi;
  if (!p || !payload || !ahat || !recon || !status || step < 1) return CF_ERR_ARG;
  if (p->dtype != CF_F32 && p->dtype != CF_BF16) return CF_ERR_ARG;
  if (p->ef != CF_EF_EXPLICIT && p->ef != CF_EF_IMPLICIT && p->ef != CF_EF_OFF) return CF_ERR_ARG;
  if (p->lr_int4 != 0 && p->lr_int4 != 1) return CF_ERR_ARG;
  if (p->iters < 1 || p->iters > 2) return CF_ERR_UNSUPPORTED;
  if (rows < 128 || cols < 128 || rows % 128 || cols % 128 || cols > kMaxCols) return CF_ERR_SHAPE;
  if (p->rank < 1 || p->rank > kMaxRank || p->rank > rows || p->rank > cols) return CF_ERR_SHAPE;
  if (((uintptr_t)payload | (uintptr_t)ahat | (uintptr_t)recon) & 15u) return CF_ERR_ALIGN;
  LowrankPlan P{};
  cf_params q = *p;
  q.role = CF_RECEIVER;
  q.batch = 1;
  lowrank_plan(rows, cols, q, &P);
  if (!P.supported) return CF_ERR_UNSUPPORTED;
  const size_t R = (size_t)rows, C = (size_t)cols, kp = (size_t)P.kp;
  const size_t need = pad256(R * kp * 2) * (P.int4 ? 1 : 2) + pad256(C * kp * 2) * 2;
  if (need > kNoAllocBytes) return CF_ERR_TOO_LARGE;
  void *scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != CF_OK) return rc;
  uint8_t *base = static_cast<uint8_t *>(scratch);
  P.b.uahi = reinterpret_cast<__nv_bfloat16 *>(base);
  base += pad256(R * kp * 2);
  if (!P.int4) {
    P.b.ualo = reinterpret_cast<__nv_bfloat16 *>(base);
    base += pad256(R * kp * 2);
  } else {
    P.b.ualo = P.b.uahi;  // not read: INT4 codes are exact in bf16
  }
  P.b.vbhi = reinterpret_cast<__nv_bfloat16 *>(base);
  base += pad256(C * kp * 2);
  P.b.vblo = reinterpret_cast<__nv_bfloat16 *>(base);
  if (!(make_map(&P.tm_uahi, P.b.uahi, kp, R, kTileM) && make_map(&P.tm_ualo, P.b.ualo, kp, R, kTileM) &&
        make_map(&P.tm_vbhi, P.b.vbhi, kp, C, kReconN) && make_map(&P.tm_vblo, P.b.vblo, kp, C, kReconN)))
    return CF_ERR_CUDA;
  // the receiver's expected header (same fields as the stateful decode)
  Header h{};
  h.w[0] = kMagic;
  h.w[1] = (uint32_t)CF_LOWRANK;
  h.w[2] = 0;
  h.w[3] = (uint32_t)p->dtype;
  h.w[4] = (uint32_t)(step & 0xffffffffu);
  h.w[5] = (uint32_t)(step >> 32);
  h.w[6] = (uint32_t)((uint64_t)rows & 0xffffffffu);
  h.w[7] = (uint32_t)((uint64_t)rows >> 32);
  h.w[8] = (uint32_t)((uint64_t)cols & 0xffffffffu);
  h.w[9] = (uint32_t)((uint64_t)cols >> 32);
  h.w[10] = 1;
  h.w[11] = (uint32_t)p->rank;
  h.w[12] = (uint32_t)p->lr_int4;
  h.w[13] = (uint32_t)p->ef;
  h.w[14] = (uint32_t)p->iters;
  h.w[15] = 0;
  const cudaError_t e = dequant_and_recon(P, static_cast<const uint8_t *>(payload), true, h, nullptr, ahat, nullptr,
                                          recon, status, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return CF_ERR_CUDA;
  }
  return CF_OK;
}
