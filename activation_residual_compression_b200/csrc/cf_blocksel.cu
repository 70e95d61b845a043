// cf_blocksel.cu -- kernels of the block-selection mode (Otil page:
// "Informative sub-block selection", "Dynamic round-robin").
//
// The state (the sender's previous activation, the receiver's values) is
// kept in the activation dtype: it only ever holds raw activations, which that
// dtype represents exactly.
//
// Encode = two launches on the caller's stream:
//   bs_encode_kernel   one CTA per (block, token row of the block): the fp64
//                      Frobenius sums <p, a>, ||p||^2, ||a||^2 and a changed
//                      flag over the row's b tokens x all channels, and the
//                      state update p = a (the row is read once); the CTA
//                      that finishes last runs the selection: d per block
//                      from the partials (fixed order), the unsent blocks
//                      ordered by (d desc, index asc) (all pairs compared
//                      when K <= 256, else a bitonic sort), the first
//                      min(k, unsent) in ascending order, the round-robin
//                      flags, the payload header and index section;
//   bs_pack_kernel     one CTA per (slot, token-row quarter): raw block rows
//                      into the payload (unused slots zeroed).
// Decode = one launch: bs_decode_kernel, one CTA per (block, token row): the
// row comes from the payload when its block was sent, else from ahat; ahat
// and recon are written.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "cf.h"
#include "cf_blocksel.h"
#include "cf_launch.cuh"

namespace cfi {
namespace {

constexpr int kBsThreads = 256;

size_t pad16(size_t x) { return (x + 15u) & ~(size_t)15u; }
size_t pad256(size_t x) { return (x + 255u) & ~(size_t)255u; }

// 8 consecutive activations as fp32, and their raw bits
template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw load(const __nv_bfloat16 *p) { return *reinterpret_cast<const uint4 *>(p); }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const Raw &r) { *reinterpret_cast<uint4 *>(p) = r; }
  static __device__ __forceinline__ void to_f32(const Raw &r, float (&x)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  // fp32 values that are bf16 numbers (received raw values): exact conversion
  static __device__ __forceinline__ Raw from_f32(const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; i++)
      w[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x[2 * i])) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x[2 * i + 1])) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Vec8<float> {
  struct Raw {
    float4 a, b;
  };
  static __device__ __forceinline__ Raw load(const float *p) {
    return Raw{reinterpret_cast<const float4 *>(p)[0], reinterpret_cast<const float4 *>(p)[1]};
  }
  static __device__ __forceinline__ void store(float *p, const Raw &r) {
    reinterpret_cast<float4 *>(p)[0] = r.a;
    reinterpret_cast<float4 *>(p)[1] = r.b;
  }
  static __device__ __forceinline__ void to_f32(const Raw &r, float (&x)[8]) {
    x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
    x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
  }
  static __device__ __forceinline__ Raw from_f32(const float (&x)[8]) {
    return Raw{make_float4(x[0], x[1], x[2], x[3]), make_float4(x[4], x[5], x[6], x[7])};
  }
};

// first token of row y of block i (the row's b tokens are consecutive)
__device__ __forceinline__ int64_t block_row_token(int i, int y, int W, int b) {
  const int nbx = W / b;
  const int by = i / nbx, bx = i - by * nbx;
  return (int64_t)(by * b + y) * W + (int64_t)bx * b;
}

// ------------------------------------------------------------------ encode

// Device-scope acquire-release fetch-and-add.
__device__ __forceinline__ unsigned atomic_add_acq_rel(unsigned *p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Order-preserving key of a double (larger d -> larger key); 0 marks "not a
// candidate" (no finite d maps to it).
__device__ __forceinline__ unsigned long long sort_key(double d) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(d);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// entry x goes before entry y: larger dissimilarity, then lower block index
__device__ __forceinline__ bool before(unsigned long long kx, int ix, unsigned long long ky, int iy) {
  return kx > ky || (kx == ky && ix < iy);
}

// d of block i from its b row partials, added in row order: 0 when every
// value is unchanged, 1 when exactly one of the two norms is zero, else
// 1 - <p, a> / (||p|| ||a||).  The partials were written by other CTAs of
// this grid: read through L2.
__device__ double block_dissimilarity(const double *part, int i, int b) {
  const double4 *src = reinterpret_cast<const double4 *>(part) + (int64_t)i * b;
  double dot = 0.0, np_ = 0.0, na = 0.0, ch = 0.0;
  for (int r0 = 0; r0 < b; r0 += 8) {
    double4 v[8];
#pragma unroll
    for (int u = 0; u < 8; u++) {
      v[u] = make_double4(0.0, 0.0, 0.0, 0.0);
      if (r0 + u < b) {
        const double2 *q2 = reinterpret_cast<const double2 *>(src + r0 + u);
        const double2 lo = __ldcg(q2), hi = __ldcg(q2 + 1);
        v[u] = make_double4(lo.x, lo.y, hi.x, hi.y);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; u++)
      if (r0 + u < b) {
        dot += v[u].x;
        np_ += v[u].y;
        na += v[u].z;
        ch = fmax(ch, v[u].w);
      }
  }
  if (ch == 0.0) return 0.0;                     // every value unchanged
  if (np_ == 0.0 || na == 0.0) return 1.0;       // exactly one zero norm
  return 1.0 - dot / (sqrt(np_) * sqrt(na));
}

// The selection, run by one CTA of kBsThreads threads once every partial is
// written: d per unsent block, the unsent blocks ordered by (d desc, index
// asc) -- for K2 <= kBsThreads each thread ranks one block against all
// others, else a bitonic sort of K2 (a power of two) entries -- the first
// min(k, unsent) blocks in ascending order into sel and the payload's index
// section, the round-robin flags (restarting the round when all are sent)
// and the payload header.
__device__ void select_blocks(const double *part, int K, int K2, int b, int k, uint8_t *sent, uint32_t *sel,
                              uint8_t *payload, const Header &hdr, uint8_t *smem) {
  unsigned long long *key = reinterpret_cast<unsigned long long *>(smem);  // [K2]
  int *idx = reinterpret_cast<int *>(key + K2);                           // [K2]
  uint8_t *pick = reinterpret_cast<uint8_t *>(idx + K2);                  // [K2]
  __shared__ int wsum[kBsThreads / 32];
  const int tid = threadIdx.x;
  for (int i = tid; i < K2; i += kBsThreads) {
    // 0 marks "not a candidate": sent in this round, or padding
    key[i] = (i < K && !sent[i]) ? sort_key(block_dissimilarity(part, i, b)) : 0ull;
    idx[i] = i;
    pick[i] = 0;
  }
  __syncthreads();
  if (K2 <= kBsThreads) {
    // rank of block tid among all K2 entries; candidates (key > 0) rank first
    if (tid < K2) {
      const unsigned long long kt = key[tid];
      int rank = 0;
#pragma unroll 8
      for (int j = 0; j < K2; j++) rank += before(key[j], j, kt, tid) ? 1 : 0;
      if (rank < k && kt != 0ull) pick[tid] = 1;
    }
  } else {
    for (int size = 2; size <= K2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        __syncthreads();
        for (int i = tid; i < K2; i += kBsThreads) {
          const int j = i ^ stride;
          if (j > i) {
            const bool up = (i & size) == 0;
            const bool jfirst = before(key[j], idx[j], key[i], idx[i]);
            const bool ifirst = before(key[i], idx[i], key[j], idx[j]);
            if (up ? jfirst : ifirst) {
              const unsigned long long tk = key[i];
              key[i] = key[j];
              key[j] = tk;
              const int ti = idx[i];
              idx[i] = idx[j];
              idx[j] = ti;
            }
          }
        }
      }
    }
    __syncthreads();
    // candidates sort first (key > 0); the first min(k, candidates) are picked
    for (int r = tid; r < K2; r += kBsThreads)
      if (r < k && key[r] != 0ull) pick[idx[r]] = 1;
  }
  __syncthreads();
  // ascending list of the picked blocks: each thread owns a contiguous chunk
  const int chunk = (K2 + kBsThreads - 1) / kBsThreads;
  const int c0 = tid * chunk;
  int cnt = 0;
  for (int i = c0; i < c0 + chunk && i < K2; i++) cnt += pick[i];
  const int lane = tid & 31, warp = tid >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int base = 0, m = 0;
  for (int w = 0; w < kBsThreads / 32; w++) {
    if (w < warp) base += wsum[w];
    m += wsum[w];
  }
  int pos = base + incl - cnt;
  uint32_t *slots = reinterpret_cast<uint32_t *>(payload + kHdrBytes);
  for (int i = c0; i < c0 + chunk && i < K2; i++)
    if (pick[i]) {
      sel[pos] = (uint32_t)i;
      slots[pos] = (uint32_t)i;
      pos++;
    }
  for (int j = m + tid; j < k; j += kBsThreads) {
    sel[j] = kBsNone;
    slots[j] = kBsNone;
  }
  for (int bb = 4 * k + tid; bb < (int)((4 * k + 15) & ~15); bb += kBsThreads) payload[kHdrBytes + bb] = 0;
  if (tid < 16) reinterpret_cast<uint32_t *>(payload)[tid] = hdr.w[tid];
  int all_sent = 1;
  for (int i = tid; i < K; i += kBsThreads) {
    const uint8_t f = (uint8_t)(sent[i] | pick[i]);
    sent[i] = f;
    all_sent &= f;
  }
  if (__syncthreads_and(all_sent))
    for (int i = tid; i < K; i += kBsThreads) sent[i] = 0;
}

// One CTA per (block, token row of the block): the row's Frobenius sums in
// fp64 (each product of two fp32 values is exact, so each fused
// multiply-add rounds once; the CTA adds its threads' sums in a fixed
// order) and the state update prev = a (the row is read once).  The CTA
// that finishes last (an acquire-release atomic count) then runs the
// selection on the complete set of partials, still in L2.
template <typename T>
__global__ void __launch_bounds__(kBsThreads) bs_encode_kernel(const T *a, T *prev, int W, int b, int64_t cols,
                                                                int K, int K2, int k, double *part,
                                                                unsigned *counter, uint8_t *sent, uint32_t *sel,
                                                                uint8_t *payload, const Header hdr) {
  pdl_enter();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int last;
  const int i = blockIdx.x / b, y = blockIdx.x - (blockIdx.x / b) * b;
  const int64_t e0 = block_row_token(i, y, W, b) * cols;
  const int64_t n8 = (int64_t)b * cols / 8;
  double dot = 0.0, np_ = 0.0, na = 0.0;
  int changed = 0;
  constexpr int U = 4;  // vectors in flight per thread
  for (int64_t v0 = threadIdx.x; v0 < n8; v0 += (int64_t)U * kBsThreads) {
    typename Vec8<T>::Raw ra[U], rp[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = v0 + (int64_t)u * kBsThreads;
      if (v < n8) {
        ra[u] = Vec8<T>::load(a + e0 + v * 8);
        rp[u] = Vec8<T>::load(prev + e0 + v * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = v0 + (int64_t)u * kBsThreads;
      if (v < n8) {
        float x[8], p[8];
        Vec8<T>::to_f32(ra[u], x);
        Vec8<T>::to_f32(rp[u], p);
#pragma unroll
        for (int q = 0; q < 8; q++) {
          changed |= p[q] != x[q];
          dot = fma((double)p[q], (double)x[q], dot);
          np_ = fma((double)p[q], (double)p[q], np_);
          na = fma((double)x[q], (double)x[q], na);
        }
        Vec8<T>::store(prev + e0 + v * 8, ra[u]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    np_ += __shfl_xor_sync(0xffffffffu, np_, o);
    na += __shfl_xor_sync(0xffffffffu, na, o);
    changed |= __shfl_xor_sync(0xffffffffu, changed, o);
  }
  __shared__ double ws[kBsThreads / 32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    ws[warp][0] = dot;
    ws[warp][1] = np_;
    ws[warp][2] = na;
    ws[warp][3] = changed ? 1.0 : 0.0;
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    double sacc = ws[0][threadIdx.x];
    for (int w = 1; w < kBsThreads / 32; w++)
      sacc = threadIdx.x == 3 ? fmax(sacc, ws[w][3]) : sacc + ws[w][threadIdx.x];
    part[(int64_t)blockIdx.x * 4 + threadIdx.x] = sacc;
  }
  // The last CTA to finish selects.  The count is an acquire-release atomic
  // after the CTA barrier: it releases this CTA's partial (the barrier orders
  // the writing threads before thread 0), and the last CTA's acquires every
  // other CTA's; the selection then reads the partials through L2.
  __syncthreads();
  if (threadIdx.x == 0) last = atomic_add_acq_rel(counter, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  select_blocks(part, K, K2, b, k, sent, sel, payload, hdr, smem);
  if (threadIdx.x == 0) *counter = 0u;  // for the next step
}

constexpr int kPackSplit = 4;  // CTAs per (slot, token row)
template <typename T>
__global__ void __launch_bounds__(kBsThreads) bs_pack_kernel(const T *a, const uint32_t *sel, int W, int b,
                                                              int64_t cols, T *data) {
  pdl_enter();
  const int row = blockIdx.x / kPackSplit, piece = blockIdx.x - row * kPackSplit;
  const int j = row / b, y = row - (row / b) * b;
  const uint32_t blk = sel[j];
  const int64_t n8 = (int64_t)b * cols / 8;
  const int64_t v0 = n8 * piece / kPackSplit, v1 = n8 * (piece + 1) / kPackSplit;
  T *dst = data + ((int64_t)j * b * b + (int64_t)y * b) * cols;
  if (blk == kBsNone) {
    float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const typename Vec8<T>::Raw zr = Vec8<T>::from_f32(z);
    for (int64_t v = v0 + threadIdx.x; v < v1; v += kBsThreads) Vec8<T>::store(dst + v * 8, zr);
    return;
  }
  const T *src = a + block_row_token((int)blk, y, W, b) * cols;
  constexpr int U = 4;  // vectors in flight per thread
  for (int64_t v0t = v0 + threadIdx.x; v0t < v1; v0t += (int64_t)U * kBsThreads) {
    typename Vec8<T>::Raw r[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = v0t + (int64_t)u * kBsThreads;
      if (v < v1) r[u] = Vec8<T>::load(src + v * 8);
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = v0t + (int64_t)u * kBsThreads;
      if (v < v1) Vec8<T>::store(dst + v * 8, r[u]);
    }
  }
}

// Full-size leading steps: payload body = a, state = a (sender); state =
// recon = body (receiver, after the header check).
template <typename T>
__global__ void __launch_bounds__(kBsThreads) bs_warm_encode_kernel(const T *a, T *prev, uint8_t *payload, int64_t E,
                                                                     const Header hdr) {
  pdl_enter();
  if (blockIdx.x == 0 && threadIdx.x < 16) reinterpret_cast<uint32_t *>(payload)[threadIdx.x] = hdr.w[threadIdx.x];
  T *body = reinterpret_cast<T *>(payload + kHdrBytes);
  const int64_t n8 = E / 8;
  for (int64_t v = (int64_t)blockIdx.x * kBsThreads + threadIdx.x; v < n8; v += (int64_t)gridDim.x * kBsThreads) {
    const typename Vec8<T>::Raw r = Vec8<T>::load(a + v * 8);
    Vec8<T>::store(body + v * 8, r);
    Vec8<T>::store(prev + v * 8, r);
  }
}

template <typename T>
__global__ void __launch_bounds__(kBsThreads) bs_warm_decode_kernel(const uint8_t *payload, T *ahat, T *recon,
                                                                     int64_t E, const Header expect, int *status) {
  pdl_enter();
  int bad = 0;
  if (threadIdx.x < 16) bad = reinterpret_cast<const uint32_t *>(payload)[threadIdx.x] != expect.w[threadIdx.x];
  if (__syncthreads_or(bad)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, 1);
    return;
  }
  const T *body = reinterpret_cast<const T *>(payload + kHdrBytes);
  const int64_t n8 = E / 8;
  for (int64_t v = (int64_t)blockIdx.x * kBsThreads + threadIdx.x; v < n8; v += (int64_t)gridDim.x * kBsThreads) {
    const typename Vec8<T>::Raw r = Vec8<T>::load(body + v * 8);
    Vec8<T>::store(ahat + v * 8, r);
    Vec8<T>::store(recon + v * 8, r);
  }
}

// ------------------------------------------------------------------ decode

template <typename T>
__global__ void __launch_bounds__(kBsThreads) bs_decode_kernel(const uint8_t *payload, T *ahat, T *recon, int W,
                                                                int b, int64_t cols, int k, int K,
                                                                const Header expect, int *status) {
  pdl_enter();
  __shared__ int slot;
  const int i = blockIdx.x / b, y = blockIdx.x - (blockIdx.x / b) * b;
  int bad = 0;
  if (threadIdx.x < 16) bad = reinterpret_cast<const uint32_t *>(payload)[threadIdx.x] != expect.w[threadIdx.x];
  if (threadIdx.x == 0) slot = -1;
  if (__syncthreads_or(bad)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, 1);
    return;
  }
  // the slot of block i in the index list (each index appears at most once)
  const uint32_t *slots = reinterpret_cast<const uint32_t *>(payload + kHdrBytes);
  for (int j = threadIdx.x; j < k; j += kBsThreads)
    if (slots[j] == (uint32_t)i && i < K) atomicMax(&slot, j);
  __syncthreads();
  const int64_t n8 = (int64_t)b * cols / 8;
  const int64_t e0 = block_row_token(i, y, W, b) * cols;
  // the row comes from the payload (its block was sent) or from ahat
  const bool from_payload = slot >= 0;
  const T *src = from_payload ? reinterpret_cast<const T *>(payload + kHdrBytes + ((4 * (size_t)k + 15) & ~(size_t)15)) +
                                    ((int64_t)slot * b * b + (int64_t)y * b) * cols
                              : ahat + e0;
  constexpr int U = 4;  // vectors in flight per thread
  for (int64_t v0 = threadIdx.x; v0 < n8; v0 += (int64_t)U * kBsThreads) {
    typename Vec8<T>::Raw r[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = v0 + (int64_t)u * kBsThreads;
      if (v < n8) r[u] = Vec8<T>::load(src + v * 8);
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = v0 + (int64_t)u * kBsThreads;
      if (v < n8) {
        if (from_payload) Vec8<T>::store(ahat + e0 + v * 8, r[u]);
        Vec8<T>::store(recon + e0 + v * 8, r[u]);
      }
    }
  }
}

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

size_t select_smem(int K2) { return (size_t)K2 * (8 + 4 + 1); }

unsigned warm_grid(int64_t E) {
  const int64_t n = (E / 8 + kBsThreads - 1) / kBsThreads;
  return (unsigned)(n < 148 * 8 ? (n > 0 ? n : 1) : 148 * 8);
}

}  // namespace

int blocksel_plan(int64_t rows, int64_t cols, int dtype, int batch, int grid_h, int block, int k, int warm,
                  BlockselPlan *P) {
  if (batch != 1) return CF_ERR_UNSUPPORTED;
  if (block != 4 && block != 8 && block != 16) return CF_ERR_UNSUPPORTED;
  if (warm < 1) return CF_ERR_ARG;
  int64_t h = grid_h;
  if (h == 0) {  // square grid
    h = 1;
    while ((h + 1) * (h + 1) <= rows) h++;
    if (h * h != rows) return CF_ERR_SHAPE;
  }
  if (h < 1 || rows % h) return CF_ERR_SHAPE;
  const int64_t w = rows / h;
  if (h % block || w % block) return CF_ERR_SHAPE;
  const int64_t K = (h / block) * (w / block);
  if (K < 1 || K > kBsMaxBlocks) return CF_ERR_UNSUPPORTED;
  const int kk = k == 0 ? (int)(K / 4 > 0 ? K / 4 : 1) : k;
  if (kk < 1 || kk > K) return CF_ERR_ARG;
  P->rows = rows;
  P->cols = cols;
  P->H = (int)h;
  P->W = (int)w;
  P->b = block;
  P->K = (int)K;
  P->k = kk;
  P->warm = warm;
  P->dtype = dtype;
  return CF_OK;
}

size_t blocksel_body_bytes(const BlockselPlan &P) {
  const size_t asz = P.dtype == CF_BF16 ? 2u : 4u;
  return pad16((size_t)P.k * 4u) + (size_t)P.k * P.b * P.b * (size_t)P.cols * asz;
}

size_t blocksel_scratch_bytes(const BlockselPlan &P) {
  return pad256((size_t)P.K) + pad256((size_t)P.K * P.b * 4 * 8) + pad256((size_t)P.k * 4) + 256;
}

int blocksel_bind(BlockselPlan *P, void *scratch) {
  uint8_t *p = static_cast<uint8_t *>(scratch);
  P->sent = p;
  p += pad256((size_t)P->K);
  P->part = reinterpret_cast<double *>(p);
  p += pad256((size_t)P->K * P->b * 4 * 8);
  P->sel = reinterpret_cast<uint32_t *>(p);
  p += pad256((size_t)P->k * 4);
  P->counter = reinterpret_cast<unsigned *>(p);
  const int sm = (int)select_smem(next_pow2(P->K));
  if (cudaFuncSetAttribute(bs_encode_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) !=
          cudaSuccess ||
      cudaFuncSetAttribute(bs_encode_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess) {
    (void)cudaGetLastError();
    return CF_ERR_CUDA;
  }
  return CF_OK;
}

namespace {

template <typename T>
cudaError_t encode_t(const BlockselPlan &P, const T *a, T *prev, uint8_t *payload, const Header &hdr,
                     cudaStream_t st) {
  const int K2 = next_pow2(P.K);
  launch_pdl(bs_encode_kernel<T>, dim3((unsigned)(P.K * P.b)), dim3(kBsThreads), select_smem(K2), st, a, prev, P.W,
             P.b, P.cols, P.K, K2, P.k, P.part, P.counter, P.sent, P.sel, payload, hdr);
  T *data = reinterpret_cast<T *>(payload + kHdrBytes + pad16((size_t)P.k * 4u));
  launch_pdl(bs_pack_kernel<T>, dim3((unsigned)(P.k * P.b * kPackSplit)), dim3(kBsThreads), 0, st, a,
             (const uint32_t *)P.sel, P.W, P.b, P.cols, data);
  return cudaGetLastError();
}

}  // namespace

cudaError_t blocksel_encode(const BlockselPlan &P, const void *a, void *prev, uint8_t *payload, const Header &hdr,
                            bool warm, cudaStream_t st) {
  const int64_t E = P.rows * P.cols;
  if (P.dtype == CF_BF16) {
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(a);
    __nv_bfloat16 *pv = static_cast<__nv_bfloat16 *>(prev);
    if (warm) {
      launch_pdl(bs_warm_encode_kernel<__nv_bfloat16>, dim3(warm_grid(E)), dim3(kBsThreads), 0, st, x, pv, payload, E, hdr);
      return cudaGetLastError();
    }
    return encode_t(P, x, pv, payload, hdr, st);
  }
  const float *x = static_cast<const float *>(a);
  float *pv = static_cast<float *>(prev);
  if (warm) {
    launch_pdl(bs_warm_encode_kernel<float>, dim3(warm_grid(E)), dim3(kBsThreads), 0, st, x, pv, payload, E, hdr);
    return cudaGetLastError();
  }
  return encode_t(P, x, pv, payload, hdr, st);
}

cudaError_t blocksel_decode(const BlockselPlan &P, const uint8_t *payload, void *ahat, void *recon,
                            const Header &expect, bool warm, int *status, cudaStream_t st) {
  const int64_t E = P.rows * P.cols;
  const unsigned grid = (unsigned)(P.K * P.b);
  if (P.dtype == CF_BF16) {
    __nv_bfloat16 *h = static_cast<__nv_bfloat16 *>(ahat), *r = static_cast<__nv_bfloat16 *>(recon);
    if (warm)
      launch_pdl(bs_warm_decode_kernel<__nv_bfloat16>, dim3(warm_grid(E)), dim3(kBsThreads), 0, st, payload, h, r, E,
                 expect, status);
    else
      launch_pdl(bs_decode_kernel<__nv_bfloat16>, dim3(grid), dim3(kBsThreads), 0, st, payload, h, r, P.W, P.b, P.cols,
                 P.k, P.K, expect, status);
    return cudaGetLastError();
  }
  float *h = static_cast<float *>(ahat), *r = static_cast<float *>(recon);
  if (warm)
    launch_pdl(bs_warm_decode_kernel<float>, dim3(warm_grid(E)), dim3(kBsThreads), 0, st, payload, h, r, E, expect,
               status);
  else
    launch_pdl(bs_decode_kernel<float>, dim3(grid), dim3(kBsThreads), 0, st, payload, h, r, P.W, P.b, P.cols, P.k, P.K,
               expect, status);
  return cudaGetLastError();
}

}  // namespace cfi
