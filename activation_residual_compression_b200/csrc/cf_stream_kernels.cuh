// cf_stream_kernels.cuh -- fused streaming kernels of the residual codec on sm_100a.
//
// Method: "Accelerating Parallel Diffusion Model Serving with Residual
// Compression" (NeurIPS 2025 paper notes).  One encode launch per step fuses
// residual formation ("Overall framework"), the error-feedback term ("Key
// design: error feedback"), the encoder (1-bit / 2-bit quantiser of the
// experiments table, or the N:M block sparsifier of "Key design: system
// co-design") and the sender-side reconstruction:
//     D = (a - ahat) + e;  payload = enc(D);  C = dec(payload)
//     e = D - C;           ahat = ahat + C
// One decode launch rebuilds the receiver's ahat from the payload and writes
// recon = cast(ahat).  The first step ("Limitations": no history) sends the
// raw activation.
//
// Mapping: a team of 2^team_log2 (>= 32) threads owns one row; thread t of
// the team holds 8-element vectors v = t + j * TEAM (j < VPT) in registers,
// so each load instruction of a warp covers 512 (bf16) or 1024 (fp32)
// contiguous bytes.  The whole row stays in registers between the row
// statistic (warp shuffles + one shared-memory stage across the team's
// warps) and the encode, so a, ahat and e are read from HBM exactly once
// and ahat, e and the payload written exactly once.  Blocks stride over row
// groups (persistent grid sized from the occupancy and the SM count).
//
// Every fp32 operation of the recurrence is an explicit round-to-nearest
// intrinsic (no contraction), so payloads and states are bit-identical to a
// scalar IEEE implementation of the same definitions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "cf_internal.h"
#include "cf_launch.cuh"

// Resident blocks per SM the compiler must allow (register budget), measured
// on B200: the decode kernels take 4 for N:M with two kept values per block
// and 3 otherwise; the encode kernels take 3 for the 1-bit and 2-bit modes and
// for up to two vectors per thread, else 2 (EncMinBlocks below).

namespace cfi {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- activations

template <typename T>
struct Act;

template <>
struct Act<float> {
  struct Raw {
    float4 lo, hi;
  };
  static __device__ __forceinline__ Raw load(const float *p) {
    const float4 *q = reinterpret_cast<const float4 *>(p);
    return Raw{__ldcs(q), __ldcs(q + 1)};
  }
  static __device__ __forceinline__ void to_f32(const Raw &r, float (&x)[8]) {
    x[0] = r.lo.x; x[1] = r.lo.y; x[2] = r.lo.z; x[3] = r.lo.w;
    x[4] = r.hi.x; x[5] = r.hi.y; x[6] = r.hi.z; x[7] = r.hi.w;
  }
  static __device__ __forceinline__ void store_raw(float *p, const Raw &r) {
    float4 *q = reinterpret_cast<float4 *>(p);
    __stcs(q, r.lo);
    __stcs(q + 1, r.hi);
  }
  static __device__ __forceinline__ void store_f32(float *p, const float (&x)[8]) {
    float4 *q = reinterpret_cast<float4 *>(p);
    __stcs(q, make_float4(x[0], x[1], x[2], x[3]));
    __stcs(q + 1, make_float4(x[4], x[5], x[6], x[7]));
  }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return a | (b << 16);
}

template <>
struct Act<__nv_bfloat16> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw load(const __nv_bfloat16 *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
  }
  // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 bits.
  static __device__ __forceinline__ void to_f32(const Raw &r, float (&x)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void store_raw(__nv_bfloat16 *p, const Raw &r) {
    __stcs(reinterpret_cast<uint4 *>(p), r);
  }
  static __device__ __forceinline__ void store_f32(__nv_bfloat16 *p, const float (&x)[8]) {
    uint4 r;
    r.x = pack_bf16x2(x[0], x[1]);
    r.y = pack_bf16x2(x[2], x[3]);
    r.z = pack_bf16x2(x[4], x[5]);
    r.w = pack_bf16x2(x[6], x[7]);
    __stcs(reinterpret_cast<uint4 *>(p), r);
  }
};

__device__ __forceinline__ void load_f32x8(const float *p, float (&x)[8]) {
  const float4 *q = reinterpret_cast<const float4 *>(p);
  float4 a = __ldcs(q), b = __ldcs(q + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void store_f32x8(float *p, const float (&x)[8]) {
  float4 *q = reinterpret_cast<float4 *>(p);
  __stcs(q, make_float4(x[0], x[1], x[2], x[3]));
  __stcs(q + 1, make_float4(x[4], x[5], x[6], x[7]));
}

// The codec state (ahat, e) is fp32, or bf16 when the caller asks for the
// bf16-state option: loads widen exactly, stores round to nearest even.
template <typename S>
__device__ __forceinline__ void load_state8(const S *p, float4 (&r)[2]) {
  float x[8];
  Act<S>::to_f32(Act<S>::load(p), x);
  r[0] = make_float4(x[0], x[1], x[2], x[3]);
  r[1] = make_float4(x[4], x[5], x[6], x[7]);
}
template <typename S>
__device__ __forceinline__ void store_state8(S *p, const float (&x)[8]) {
  Act<S>::store_f32(p, x);
}

template <typename T, typename Tab>
__device__ __forceinline__ const T *act_tensor(const void *base, const Tab &tab, int64_t b, int64_t E);
template <>
__device__ __forceinline__ const float *act_tensor<float, NoTable>(const void *base, const NoTable &, int64_t b,
                                                                    int64_t E) {
  return static_cast<const float *>(base) + b * E;
}
template <>
__device__ __forceinline__ const __nv_bfloat16 *act_tensor<__nv_bfloat16, NoTable>(const void *base, const NoTable &,
                                                                                    int64_t b, int64_t E) {
  return static_cast<const __nv_bfloat16 *>(base) + b * E;
}
template <>
__device__ __forceinline__ const float *act_tensor<float, PtrTable>(const void *, const PtrTable &tab, int64_t b,
                                                                     int64_t) {
  return static_cast<const float *>(tab.p[b]);
}
template <>
__device__ __forceinline__ const __nv_bfloat16 *act_tensor<__nv_bfloat16, PtrTable>(const void *, const PtrTable &tab,
                                                                                     int64_t b, int64_t) {
  return static_cast<const __nv_bfloat16 *>(tab.p[b]);
}

// ---------------------------------------------------------------- reductions

// Max over the team (all threads of the block call this together).
// Barrier of one team only (named barrier 1 + team index; a block holds at
// most kBlock / 64 = 4 multi-warp teams), so that the teams of a block do not
// wait for one another.
static_assert(kBlock / 64 <= 15, "named team barriers use ids 1 .. kBlock / 64");
__device__ __forceinline__ void team_bar(int team_log2) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + (int)(threadIdx.x >> team_log2)), "r"(1 << team_log2) : "memory");
}

__device__ __forceinline__ float team_max(float x, int team_log2, float *sm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
  if (team_log2 > 5) {
    const int warp = threadIdx.x >> 5, wpt = 1 << (team_log2 - 5);
    if ((threadIdx.x & 31) == 0) sm[warp] = x;
    team_bar(team_log2);
    const int w0 = warp & ~(wpt - 1);
    x = sm[w0];
    for (int w = 1; w < wpt; w++) x = fmaxf(x, sm[w0 + w]);
    team_bar(team_log2);
  }
  return x;
}

__device__ __forceinline__ unsigned long long team_sum_u64(unsigned long long x, int team_log2,
                                                           unsigned long long *sm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
  if (team_log2 > 5) {
    const int warp = threadIdx.x >> 5, wpt = 1 << (team_log2 - 5);
    if ((threadIdx.x & 31) == 0) sm[warp] = x;
    team_bar(team_log2);
    const int w0 = warp & ~(wpt - 1);
    x = sm[w0];
    for (int w = 1; w < wpt; w++) x += sm[w0 + w];
    team_bar(team_log2);
  }
  return x;
}

// OR over aligned groups of G consecutive lanes (G a power of two <= 32).
template <int G>
__device__ __forceinline__ uint32_t group_or(uint32_t x) {
#pragma unroll
  for (int o = 1; o < G; o <<= 1) x |= __shfl_xor_sync(kFull, x, o);
  return x;
}

// ---------------------------------------------------------------- SIGN1 scale

// Fraction bits of the 1-bit scale's fixed-point sum, below the row
// maximum's leading bit: q_i = floor(|d_i| 2^(31-E)) < 2^32.
constexpr int kFxF = 31;

// floor(ad * 2^sh_base) for a non-negative finite fp32 ad, exactly, from its
// bits (used when 2^sh_base is not a normal fp32; ad < 2^(E+1) keeps the
// result below 2^32).
__device__ __forceinline__ unsigned long long fixed_term(float ad, int sh_base) {
  const uint32_t bits = __float_as_uint(ad);
  int e = int(bits >> 23);
  uint32_t mant = bits & 0x7fffffu;
  if (e) mant |= 0x800000u; else e = 1;
  const int sh = e - 150 + sh_base;
  if (sh >= 0) return (unsigned long long)mant << sh;
  const int rs = -sh;
  return rs >= 24 ? 0ull : (unsigned long long)(mant >> rs);
}

// floor(log2 m) for a finite m > 0.
__device__ __forceinline__ int floor_log2_f32(float m) {
  const uint32_t bits = __float_as_uint(m);
  const int e = int(bits >> 23);
  if (e) return e - 127;
  return (31 - __clz(bits & 0x7fffffu)) - 149;
}

// ---------------------------------------------------------------- Q2 helpers

// Levels ((2q-3) S) / 3 for q = 0..3, each exactly as that expression
// rounds: (3S)/3 is S unless 3S overflows to infinity, and (-S)/3 = -(S/3).
__device__ __forceinline__ void q2_levels(float S, float (&L)[4]) {
  const float third = __fdiv_rn(S, 3.0f);
  const float full = isinf(__fmul_rn(3.0f, S)) ? __int_as_float(0x7f800000) : S;
  L[0] = -full;
  L[1] = -third;
  L[2] = third;
  L[3] = full;
}

// Code q = rint(clamp(u, 0, 3)) with u = RN(RN(RN(d/S) * 1.5) + 1.5) (S != 0),
// returned as a float in {0, 1, 2, 3}.
// u_a = fma(d, RN(1.5/S), 1.5) is within 2^-20.9 of u for |d| <= 1.01 S, so
// when u_a is at least 2^-20 away from every decision boundary (0.5, 1.5,
// 2.5) both fall in the same interval and give the same code; otherwise the
// exact division chain decides.
__device__ __forceinline__ float q2_code(float d, float S, float k1) {
  const float ua = __fmaf_rn(d, k1, 1.5f);
  const float qa = rintf(fminf(fmaxf(ua, 0.0f), 3.0f));
  if (fabsf(__fsub_rn(ua, qa)) <= 0.5f - 0x1p-20f) return qa;
  float u = __fmul_rn(__fdiv_rn(d, S), 1.5f);
  u = __fadd_rn(u, 1.5f);
  u = fminf(fmaxf(u, 0.0f), 3.0f);
  return rintf(u);
}

// Level of code q (as a float in {0,1,2,3}): sign from q - 1.5, magnitude
// `full` for q in {0, 3} and `third` for q in {1, 2} (see q2_levels).
__device__ __forceinline__ float q2_level(float qf, float third, float full) {
  const float t = __fsub_rn(qf, 1.5f);
  const float mag = fabsf(t) > 1.0f ? full : third;
  return copysignf(mag, t);
}

// Integer value of a float in {0, 1, 2, 3}: the low bits of qf + 2^23.
__device__ __forceinline__ uint32_t small_uint(float qf) { return __float_as_uint(__fadd_rn(qf, 8388608.0f)) & 3u; }

// ---------------------------------------------------------------- mode traits

enum { M_ID = CF_IDENTITY, M_S1 = CF_SIGN1, M_Q2 = CF_Q2, M_NM = CF_NM };

// Bits of packed code per 8-element vector, and lanes per payload word.
template <int MODE, int NM_M, int NM_N>
struct Pack {
  static constexpr int bpv = MODE == M_S1 ? 8 : MODE == M_Q2 ? 16 : MODE == M_NM ? (NM_M == 16 ? 2 * NM_N : 4 * NM_N) : 0;
  static constexpr int G = bpv ? 32 / bpv : 1;
};

// Top-N (N <= 2) of |x[k]| over k in [k0, k0+cnt), key (|x| desc, index asc).
template <int N>
__device__ __forceinline__ void local_topn(const float (&x)[8], int k0, int cnt, float (&bv)[2], int (&bi)[2]) {
  bv[0] = -1.0f; bv[1] = -1.0f; bi[0] = 0; bi[1] = 0;
#pragma unroll
  for (int k = 0; k < cnt; k++) {  // selects, no divergent branch; strict > keeps the lower index on ties
    const float a = fabsf(x[k0 + k]);
    const bool gt0 = a > bv[0];
    const bool gt1 = N == 2 && !gt0 && a > bv[1];
    const float v1 = gt0 ? bv[0] : (gt1 ? a : bv[1]);
    const int i1 = gt0 ? bi[0] : (gt1 ? k : bi[1]);
    bv[0] = gt0 ? a : bv[0];
    bi[0] = gt0 ? k : bi[0];
    bv[1] = v1;
    bi[1] = i1;
  }
}

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) { return a > b || (a == b && ia < ib); }

// ---------------------------------------------------------------- encode

// Tensor b and row r of global row gr (32-bit division when it fits).
__device__ __forceinline__ void split_row(int64_t gr, int64_t rows, int batch, int64_t &b, int64_t &r) {
  if (batch == 1) {
    b = 0;
    r = gr;
  } else if (gr < 0x7fffffff && rows < 0x7fffffff) {
    const uint32_t q = (uint32_t)gr / (uint32_t)rows;
    b = q;
    r = gr - (int64_t)q * rows;
  } else {
    b = gr / rows;
    r = gr - b * rows;
  }
}


// The (< 16 byte) alignment padding of every tensor body is written as zero,
// so the whole payload is defined.  One thread per tensor.
__device__ __forceinline__ void zero_padding(const EncArgs &A) {
  const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < A.batch; b += nthr) {
    uint8_t *body = A.payload + kHdrBytes + b * A.body_bytes;
    for (int64_t i = 0; i < A.padA_len; i++) body[A.padA_off + i] = 0;
    for (int64_t i = 0; i < A.padB_len; i++) body[A.padB_off + i] = 0;
  }
}

// One row of the fused encode, given the thread's raw inputs (a, ahat, e of
// its vectors v = t + j * TEAM): residual with error feedback, row statistic,
// encode, payload stores, e = D - C and ahat = ahat + C stores (with
// CF_EF_OFF: ahat = fp32(a) and no e store).  Every thread
// of the team calls this together (team reductions use the team's barrier).
template <int MODE, typename T, int VPT, int NM_M, int NM_N, typename S>
__device__ __forceinline__ void encode_row(const EncArgs &A, const int t, const int tlog, const bool row_ok,
                                           const int64_t r, S *hrow, S *erow, uint8_t *body,
                                           const typename Act<T>::Raw (&ra)[VPT], const float4 (&rh)[VPT][2],
                                           const float4 (&re)[VPT][2], float *sm_f, unsigned long long *sm_u) {
  using P = Pack<MODE, NM_M, NM_N>;
  const int64_t cols = A.cols;
  const int V = (int)(cols >> 3);

  // ---- residual with error feedback: D = (a - ahat) + e ----
  float d[VPT][8], h[VPT][8];
#pragma unroll
  for (int j = 0; j < VPT; j++) {
    float x[8];
    Act<T>::to_f32(ra[j], x);
    const float hv[8] = {rh[j][0].x, rh[j][0].y, rh[j][0].z, rh[j][0].w,
                         rh[j][1].x, rh[j][1].y, rh[j][1].z, rh[j][1].w};
    const float ev[8] = {re[j][0].x, re[j][0].y, re[j][0].z, re[j][0].w,
                         re[j][1].x, re[j][1].y, re[j][1].z, re[j][1].w};
#pragma unroll
    for (int k = 0; k < 8; k++) {
      // without error feedback the new state is the activation itself; it
      // takes the registers of ahat, which the update then does not need
      h[j][k] = A.ef_off ? x[k] : hv[k];
      const float tt = __fsub_rn(x[k], hv[k]);
      d[j][k] = A.ef_explicit ? __fadd_rn(tt, ev[k]) : tt;
    }
  }

  // ---- encode; c[j][k] = C(D) from the encoded values ----
  // C(D) for the state update below, rebuilt there from compact data rather
  // than held as VPT x 8 floats: the 1-bit value from the sign of D and the
  // scale, the 2-bit value from its code and two levels, the N:M value from
  // the kept mask (fewer live registers: the 1-bit encode fits the budget of
  // three resident blocks per SM).
  float cL2 = 0.0f, cL3 = 0.0f;
  uint32_t cinfo[VPT];
  float cS1 = 0.0f;
#pragma unroll
  for (int j = 0; j < VPT; j++) cinfo[j] = 0;
  uint32_t cbits[VPT];
#pragma unroll
  for (int j = 0; j < VPT; j++) cbits[j] = 0;

  if constexpr (MODE == M_ID) {
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      if (row_ok && v < V) store_f32x8(reinterpret_cast<float *>(body) + r * cols + v * 8, d[j]);
    }
  } else if constexpr (MODE == M_S1) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; j++)
#pragma unroll
      for (int k = 0; k < 8; k++) m = fmaxf(m, fabsf(d[j][k]));
    m = team_max(m, tlog, sm_f);
    float Sc = 0.0f;
    unsigned long long q = 0;
    const int Ex = m > 0.0f ? floor_log2_f32(m) : 0;
    if (m > 0.0f) {
      if (Ex >= kFxF - 127) {
        // 2^(31-E) is a normal fp32: |d| * 2^(31-E) is exact (< 2^32), and the
        // truncating conversion is the floor
        const float p2 = __uint_as_float((uint32_t)(127 + kFxF - Ex) << 23);
#pragma unroll
        for (int j = 0; j < VPT; j++)
#pragma unroll
          for (int k = 0; k < 8; k++) q += __float2uint_rz(__fmul_rn(fabsf(d[j][k]), p2));
      } else {
#pragma unroll
        for (int j = 0; j < VPT; j++)
#pragma unroll
          for (int k = 0; k < 8; k++) q += fixed_term(fabsf(d[j][k]), kFxF - Ex);
      }
    }
    q = team_sum_u64(q, tlog, sm_u);
    uint16_t sbits = 0;
    if (m > 0.0f) {
      // mean = fp64(Q) * 2^(E - 31) / cols; Q < 2^53 converts exactly and the
      // power-of-two scaling is exact
      const double p2 = __hiloint2double((Ex - kFxF + 1023) << 20, 0);
      const double mean = __ddiv_rn(__dmul_rn(__ull2double_rn(q), p2), (double)cols);
      sbits = __bfloat16_as_ushort(__float2bfloat16_rn(__double2float_rn(mean)));
      Sc = __uint_as_float((uint32_t)sbits << 16);
    }
    if (row_ok && t == 0) reinterpret_cast<uint16_t *>(body)[r] = sbits;
    cS1 = Sc;
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      uint32_t byte = 0;
#pragma unroll
      for (int k = 0; k < 8; k++) {
        const bool neg = d[j][k] < 0.0f;
        byte |= (uint32_t)neg << k;
      }
      const int v = t + (j << tlog);
      cbits[j] = byte << ((v % P::G) * P::bpv);
    }
  } else if constexpr (MODE == M_Q2) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; j++)
#pragma unroll
      for (int k = 0; k < 8; k++) m = fmaxf(m, fabsf(d[j][k]));
    m = team_max(m, tlog, sm_f);
    const uint16_t sbits = __bfloat16_as_ushort(__float2bfloat16_rn(m));
    const float Sc = __uint_as_float((uint32_t)sbits << 16);
    if (row_ok && t == 0) reinterpret_cast<uint16_t *>(body)[r] = sbits;
    float L[4];
    q2_levels(Sc, L);
    cL2 = L[2];
    cL3 = L[3];
    const float k1 = Sc != 0.0f ? __fdiv_rn(1.5f, Sc) : 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      uint32_t codes = 0;
#pragma unroll
      for (int k = 0; k < 8; k++) {
        const float qf = Sc != 0.0f ? q2_code(d[j][k], Sc, k1) : 0.0f;
        codes |= small_uint(qf) << (2 * k);
      }
      cinfo[j] = codes;
      const int v = t + (j << tlog);
      cbits[j] = codes << ((v % P::G) * P::bpv);
    }
  } else {  // M_NM
    const int64_t nblk_row = cols / NM_M;
    uint16_t *vals = reinterpret_cast<uint16_t *>(body) + r * nblk_row * NM_N;
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      const bool ok = row_ok && v < V;
      if constexpr (NM_M == 16) {
        // a block of 16 columns spans the vector pair (v even, v odd) held by lanes (t, t^1)
        float bv[2];
        int bi[2];
        local_topn<NM_N>(d[j], 0, 8, bv, bi);
        const int half = int(v & 1);
        float bd[2] = {d[j][0], d[j][0]};
#pragma unroll
        for (int k = 0; k < 8; k++) {
          if (k == bi[0]) bd[0] = d[j][k];
          if (k == bi[1]) bd[1] = d[j][k];
        }
        int gi[2] = {bi[0] + 8 * half, bi[1] + 8 * half};
        float pv[2], pd[2];
        int pi[2];
#pragma unroll
        for (int s = 0; s < 2; s++) {
          pv[s] = __shfl_xor_sync(kFull, bv[s], 1);
          pd[s] = __shfl_xor_sync(kFull, bd[s], 1);
          pi[s] = __shfl_xor_sync(kFull, gi[s], 1);
        }
        // merge the two sorted candidate lists, keep the first NM_N
        int ki[2] = {0, 0};
        float kd[2] = {0.f, 0.f};
        {
          int ia = 0, ib = 0;
#pragma unroll
          for (int s = 0; s < NM_N; s++) {
            const float av = ia == 0 ? bv[0] : bv[1];
            const int ai = ia == 0 ? gi[0] : gi[1];
            const float ad = ia == 0 ? bd[0] : bd[1];
            const float bvv = ib == 0 ? pv[0] : pv[1];
            const int bii = ib == 0 ? pi[0] : pi[1];
            const float bdd = ib == 0 ? pd[0] : pd[1];
            const bool take_a = better(av, ai, bvv, bii);  // selects, no divergent branch
            ki[s] = take_a ? ai : bii;
            kd[s] = take_a ? ad : bdd;
            ia += take_a ? 1 : 0;
            ib += take_a ? 0 : 1;
          }
        }
        if (NM_N == 2) {  // ascending indices
          const bool sw = ki[0] > ki[1];
          const int i0 = sw ? ki[1] : ki[0], i1 = sw ? ki[0] : ki[1];
          const float d0 = sw ? kd[1] : kd[0], d1 = sw ? kd[0] : kd[1];
          ki[0] = i0; ki[1] = i1;
          kd[0] = d0; kd[1] = d1;
        }
#pragma unroll
        for (int k = 0; k < 8; k++) {
          const int gk = k + 8 * half;
          bool keep = gk == ki[0];
          if (NM_N == 2) keep = keep || gk == ki[1];
          if (keep) cinfo[j] |= 1u << k;
        }
        if (half == 0) {
          const int blk = v >> 1;
          uint32_t fields = 0;
#pragma unroll
          for (int s = 0; s < NM_N; s++) fields |= (uint32_t)ki[s] << (4 * s);
          cbits[j] = fields << ((v % P::G) * P::bpv);
          if (ok) {
            if (NM_N == 1) {
              vals[blk] = __bfloat16_as_ushort(__float2bfloat16_rn(kd[0]));
            } else {
              reinterpret_cast<uint32_t *>(vals)[blk] = pack_bf16x2(kd[0], kd[1]);
            }
          }
        }
      } else {  // NM_M == 4: two blocks inside the vector
        uint32_t fields = 0;
        uint16_t vb[4] = {0, 0, 0, 0};
#pragma unroll
        for (int qb = 0; qb < 2; qb++) {
          float bv[2];
          int bi[2];
          local_topn<NM_N>(d[j], 4 * qb, 4, bv, bi);
          int ki[2] = {bi[0], bi[1]};
          if (NM_N == 2) {  // ascending indices, by selects
            const bool sw = ki[0] > ki[1];
            const int i0 = sw ? ki[1] : ki[0], i1 = sw ? ki[0] : ki[1];
            ki[0] = i0; ki[1] = i1;
          }
#pragma unroll
          for (int s = 0; s < NM_N; s++) {
            float dv = d[j][4 * qb];
#pragma unroll
            for (int k = 1; k < 4; k++)
              if (k == ki[s]) dv = d[j][4 * qb + k];
            const __nv_bfloat16 bb = __float2bfloat16_rn(dv);
            vb[qb * NM_N + s] = __bfloat16_as_ushort(bb);
            fields |= (uint32_t)ki[s] << (2 * (qb * NM_N + s));
#pragma unroll
            for (int k = 0; k < 4; k++)
              if (k == ki[s]) cinfo[j] |= 1u << (4 * qb + k);
          }
        }
        cbits[j] = fields << ((v % P::G) * P::bpv);
        if (ok) {
          const int blk0 = 2 * v;
          if (NM_N == 1) {
            reinterpret_cast<uint32_t *>(vals + blk0)[0] = (uint32_t)vb[0] | ((uint32_t)vb[1] << 16);
          } else {
            uint2 w;
            w.x = (uint32_t)vb[0] | ((uint32_t)vb[1] << 16);
            w.y = (uint32_t)vb[2] | ((uint32_t)vb[3] << 16);
            reinterpret_cast<uint2 *>(vals + blk0 * 2)[0] = w;
          }
        }
      }
    }
  }

  // ---- packed code words: OR over the G lanes of a word, one store ----
  if constexpr (P::bpv > 0) {
    const int64_t W = V / P::G;
    uint32_t *words = reinterpret_cast<uint32_t *>(body + A.sec1) + r * W;
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      const uint32_t w = group_or<P::G>(cbits[j]);
      if (row_ok && v < V && (v % P::G) == 0) words[v / P::G] = w;
    }
  }

  // ---- error feedback and sender reconstruction ----
#pragma unroll
  for (int j = 0; j < VPT; j++) {
    const int v = t + (j << tlog);
    if (row_ok && v < V) {
      float c[8];
#pragma unroll
      for (int k = 0; k < 8; k++) {
        if constexpr (MODE == M_ID) c[k] = d[j][k];
        else if constexpr (MODE == M_S1) c[k] = d[j][k] < 0.0f ? -cS1 : cS1;
        else if constexpr (MODE == M_Q2) c[k] = q2_level((float)((cinfo[j] >> (2 * k)) & 3u), cL2, cL3);
        else c[k] = ((cinfo[j] >> k) & 1u) ? __bfloat162float(__float2bfloat16_rn(d[j][k])) : 0.0f;
      }
      float en[8], hn[8];
#pragma unroll
      for (int k = 0; k < 8; k++) {
        en[k] = __fsub_rn(d[j][k], c[k]);
        hn[k] = A.ef_off ? h[j][k] : __fadd_rn(h[j][k], c[k]);
      }
      if (!A.ef_off) store_state8(erow + v * 8, en);
      store_state8(hrow + v * 8, hn);
    }
  }
}

// Register path: each thread loads its vectors straight from global memory.
template <int MODE, int VPT>
struct EncMinBlocks {
  static constexpr int value = (MODE == CF_Q2 || MODE == CF_SIGN1 || VPT <= 2) ? 3 : 2;
};

template <int MODE, typename T, int VPT, int NM_M, int NM_N, typename Tab, typename S = float>
__global__ void __launch_bounds__(kBlock, EncMinBlocks<MODE, VPT>::value) encode_kernel(const EncArgs A, const __grid_constant__ Tab tab) {
  __shared__ float sm_f[kBlock / 32];
  __shared__ unsigned long long sm_u[kBlock / 32];
  const int tlog = A.team_log2;
  const int TEAM = 1 << tlog;
  const int t = threadIdx.x & (TEAM - 1);
  const int team = threadIdx.x >> tlog;
  const int tpb = kBlock >> tlog;
  const int64_t cols = A.cols;
  const int V = (int)(cols >> 3);
  const int64_t E = A.rows * cols;
  const int64_t nrows = (int64_t)A.batch * A.rows;
  const int64_t n_rg = (nrows + tpb - 1) / tpb;

  pdl_enter();  // every global access below follows the previous kernel of the stream
  if (blockIdx.x == 0 && threadIdx.x < 16) reinterpret_cast<uint32_t *>(A.payload)[threadIdx.x] = A.hdr.w[threadIdx.x];
  zero_padding(A);

  for (int64_t rg = blockIdx.x; rg < n_rg; rg += gridDim.x) {
    const int64_t gr = rg * tpb + team;
    const bool row_ok = gr < nrows;
    int64_t b = 0, r = 0;
    if (row_ok) split_row(gr, A.rows, A.batch, b, r);
    const T *arow = act_tensor<T, Tab>(A.a, tab, b, E) + r * cols;
    S *hrow = reinterpret_cast<S *>(A.ahat) + (row_ok ? gr : 0) * cols;
    S *erow = reinterpret_cast<S *>(A.err) + (row_ok ? gr : 0) * cols;
    uint8_t *body = A.payload + kHdrBytes + b * A.body_bytes;
    typename Act<T>::Raw ra[VPT];
    float4 rh[VPT][2], re[VPT][2];
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      ra[j] = typename Act<T>::Raw{};
      rh[j][0] = rh[j][1] = re[j][0] = re[j][1] = z;
      if (row_ok && v < V) {
        ra[j] = Act<T>::load(arow + v * 8);
        load_state8(hrow + v * 8, rh[j]);
        if (A.ef_explicit) load_state8(erow + v * 8, re[j]);
      }
    }
    encode_row<MODE, T, VPT, NM_M, NM_N, S>(A, t, tlog, row_ok, r, hrow, erow, body, ra, rh, re, sm_f, sm_u);
  }
}

// ---------------------------------------------------------------- decode

template <typename Tab>
__device__ __forceinline__ void *recon_tensor(void *base, const Tab &tab, int64_t b, int64_t bytes);
template <>
__device__ __forceinline__ void *recon_tensor<NoTable>(void *base, const NoTable &, int64_t b, int64_t bytes) {
  return static_cast<uint8_t *>(base) + b * bytes;
}
template <>
__device__ __forceinline__ void *recon_tensor<PtrTable>(void *, const PtrTable &tab, int64_t b, int64_t) {
  return const_cast<void *>(tab.p[b]);
}

// Compare the payload header with the expected one; on a mismatch record the
// status (block 0) and tell the caller to return.
__device__ __forceinline__ bool header_ok(const DecArgs &A) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  if (threadIdx.x < 16) {
    const uint32_t w = reinterpret_cast<const uint32_t *>(A.payload)[threadIdx.x];
    if (w != A.expect.w[threadIdx.x]) atomicOr(&bad, 1);
  }
  __syncthreads();
  if (bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(A.status, 1);
    return false;
  }
  return true;
}

// The payload words one thread needs for its vectors of one row (identity
// mode streams its fp32 payload like the state instead).
template <int VPT>
struct DecIn {
  float S;
  uint32_t w[VPT];
  uint2 nv[VPT];
};

template <int MODE, int VPT, int NM_M, int NM_N>
__device__ __forceinline__ void load_dec_in(const DecArgs &A, const uint8_t *body, const int64_t r, const int t,
                                            const int tlog, const bool row_ok, DecIn<VPT> &in) {
  using P = Pack<MODE, NM_M, NM_N>;
  const int V = (int)(A.cols >> 3);
  in.S = 0.0f;
#pragma unroll
  for (int j = 0; j < VPT; j++) {
    in.w[j] = 0;
    in.nv[j] = make_uint2(0, 0);
  }
  if (!row_ok) return;
  if constexpr (MODE == M_S1 || MODE == M_Q2)
    in.S = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(body)[r] << 16);
  if constexpr (P::bpv > 0) {
    const int64_t W = V / P::G;
    const uint32_t *words = reinterpret_cast<const uint32_t *>(body + A.sec1) + r * W;
    const int64_t nblk_row = A.cols / (NM_M > 0 ? NM_M : 1);
    const uint16_t *vals = reinterpret_cast<const uint16_t *>(body) + r * nblk_row * NM_N;
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      if (v < V) {
        if constexpr (MODE == M_NM && NM_M == 16) {
          const int v0 = v & ~1;
          in.w[j] = __ldcs(words + v0 / P::G);
          const int blk = v >> 1;
          if constexpr (NM_N == 1) in.nv[j].x = vals[blk];
          else in.nv[j].x = __ldcs(reinterpret_cast<const uint32_t *>(vals) + blk);
        } else {
          in.w[j] = __ldcs(words + v / P::G);
          if constexpr (MODE == M_NM && NM_N == 1) in.nv[j].x = __ldcs(reinterpret_cast<const uint32_t *>(vals + 2 * v));
          if constexpr (MODE == M_NM && NM_N == 2) in.nv[j] = __ldcs(reinterpret_cast<const uint2 *>(vals + 4 * v));
        }
      }
    }
  }
}

__device__ __forceinline__ float bf16_half(uint32_t w, int hi) { return __uint_as_float(hi ? (w & 0xffff0000u) : (w << 16)); }

// One row of the decode: C from the payload, ahat = ahat + C (fp32 RN),
// recon = cast(ahat).  rp holds the identity mode's fp32 payload vectors.
template <int MODE, typename T, int VPT, int NM_M, int NM_N, typename S>
__device__ __forceinline__ void decode_row(const DecArgs &A, const int t, const int tlog, S *hrow, T *rrow,
                                           const float4 (&rh)[VPT][2], const float4 (&rp)[VPT][2],
                                           const DecIn<VPT> &in) {
  using P = Pack<MODE, NM_M, NM_N>;
  const int V = (int)(A.cols >> 3);
  float L[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (MODE == M_Q2) q2_levels(in.S, L);
#pragma unroll
  for (int j = 0; j < VPT; j++) {
    const int v = t + (j << tlog);
    if (v >= V) continue;
    float c[8];
    if constexpr (MODE == M_ID) {
      c[0] = rp[j][0].x; c[1] = rp[j][0].y; c[2] = rp[j][0].z; c[3] = rp[j][0].w;
      c[4] = rp[j][1].x; c[5] = rp[j][1].y; c[6] = rp[j][1].z; c[7] = rp[j][1].w;
    } else if constexpr (MODE == M_S1) {
      const uint32_t byte = (in.w[j] >> ((v % P::G) * P::bpv)) & 0xffu;
#pragma unroll
      for (int k = 0; k < 8; k++) c[k] = ((byte >> k) & 1u) ? -in.S : in.S;
    } else if constexpr (MODE == M_Q2) {
      const uint32_t codes = (in.w[j] >> ((v % P::G) * P::bpv)) & 0xffffu;
#pragma unroll
      for (int k = 0; k < 8; k++) {
        // level of code q: magnitude L[3] for q in {0,3}, L[2] for {1,2}; negative for q < 2
        const uint32_t qv = (codes >> (2 * k)) & 3u;
        const float mag = ((qv ^ (qv >> 1)) & 1u) ? L[2] : L[3];
        c[k] = (qv & 2u) ? mag : -mag;
      }
    } else {  // NM
#pragma unroll
      for (int k = 0; k < 8; k++) c[k] = 0.0f;
      if constexpr (NM_M == 16) {
        const int half = int(v & 1);
        const int v0 = v & ~1;
        const uint32_t fields = (in.w[j] >> ((v0 % P::G) * P::bpv)) & ((1u << (4 * NM_N)) - 1u);
#pragma unroll
        for (int s = 0; s < NM_N; s++) {
          const int idx = int((fields >> (4 * s)) & 15u);
          const float val = bf16_half(in.nv[j].x, s);
          // position in this half, or 8 (nowhere) when the kept value is in the other
          // half: selects only, no divergent branch
          const int pos = ((idx >> 3) == half) ? (idx & 7) : 8;
#pragma unroll
          for (int k = 0; k < 8; k++) c[k] = (k == pos) ? val : c[k];
        }
      } else {  // NM_M == 4
        const uint32_t fields = (in.w[j] >> ((v % P::G) * P::bpv)) & ((1u << P::bpv) - 1u);
#pragma unroll
        for (int qb = 0; qb < 2; qb++)
#pragma unroll
          for (int s = 0; s < NM_N; s++) {
            const int f = qb * NM_N + s;  // value slot 0..3
            const int idx = int((fields >> (2 * f)) & 3u);
            const float val = bf16_half(f < 2 ? in.nv[j].x : in.nv[j].y, f & 1);
#pragma unroll
            for (int k = 0; k < 4; k++)
              if (k == idx) c[4 * qb + k] = val;
          }
      }
    }
    const float hv[8] = {rh[j][0].x, rh[j][0].y, rh[j][0].z, rh[j][0].w,
                         rh[j][1].x, rh[j][1].y, rh[j][1].z, rh[j][1].w};
    float hn[8];
#pragma unroll
    for (int k = 0; k < 8; k++) hn[k] = __fadd_rn(hv[k], c[k]);
    store_state8(hrow + v * 8, hn);
    Act<T>::store_f32(rrow + v * 8, hn);  // a bf16 state and a bf16 recon round alike
  }
}

template <int MODE, int NM_N>
struct DecMinBlocks {
  static constexpr int value = (MODE == M_NM && NM_N == 2) ? 4 : 3;
};

template <int MODE, typename T, int VPT, int NM_M, int NM_N, typename Tab, typename S = float>
__global__ void __launch_bounds__(kBlock, DecMinBlocks<MODE, NM_N>::value) decode_kernel(const DecArgs A, const __grid_constant__ Tab tab) {
  pdl_enter();
  if (!header_ok(A)) return;
  const int tlog = A.team_log2;
  const int TEAM = 1 << tlog;
  const int t = threadIdx.x & (TEAM - 1);
  const int team = threadIdx.x >> tlog;
  const int tpb = kBlock >> tlog;
  const int64_t cols = A.cols;
  const int V = (int)(cols >> 3);
  const int64_t E = A.rows * cols;
  const int64_t nrows = (int64_t)A.batch * A.rows;
  const int64_t n_rg = (nrows + tpb - 1) / tpb;
  for (int64_t rg = blockIdx.x; rg < n_rg; rg += gridDim.x) {
    const int64_t gr = rg * tpb + team;
    if (gr >= nrows) continue;  // no block-wide synchronisation below
    int64_t b, r;
    split_row(gr, A.rows, A.batch, b, r);
    const uint8_t *body = A.payload + kHdrBytes + b * A.body_bytes;
    T *rrow = static_cast<T *>(recon_tensor<Tab>(A.recon, tab, b, E * (int64_t)sizeof(T))) + r * cols;
    S *hrow = reinterpret_cast<S *>(A.ahat) + gr * cols;
    DecIn<VPT> in;
    load_dec_in<MODE, VPT, NM_M, NM_N>(A, body, r, t, tlog, true, in);
    float4 rh[VPT][2], rp[VPT][2];
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      rh[j][0] = rh[j][1] = rp[j][0] = rp[j][1] = z;
      if (v < V) {
        load_state8(hrow + v * 8, rh[j]);
        if constexpr (MODE == M_ID) {
          const float4 *pp = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(body) + r * cols + v * 8);
          rp[j][0] = __ldcs(pp);
          rp[j][1] = __ldcs(pp + 1);
        }
      }
    }
    decode_row<MODE, T, VPT, NM_M, NM_N, S>(A, t, tlog, hrow, rrow, rh, rp, in);
  }
}

// ---------------------------------------------------------------- warm-up kernels

// Step 0: payload body = raw a; ahat = fp32(a); e = 0.
template <typename T, int VPT, typename Tab, typename S = float>
__global__ void __launch_bounds__(kBlock) warm_encode_kernel(const EncArgs A, const __grid_constant__ Tab tab) {
  pdl_enter();
  const int tlog = A.team_log2;
  const int TEAM = 1 << tlog;
  const int t = threadIdx.x & (TEAM - 1);
  const int team = threadIdx.x >> tlog;
  const int tpb = kBlock >> tlog;
  const int64_t cols = A.cols, E = A.rows * cols;
  const int V = (int)(cols >> 3);
  const int64_t nrows = (int64_t)A.batch * A.rows;
  const int64_t n_rg = (nrows + tpb - 1) / tpb;
  if (blockIdx.x == 0 && threadIdx.x < 16) reinterpret_cast<uint32_t *>(A.payload)[threadIdx.x] = A.hdr.w[threadIdx.x];
  for (int64_t rg = blockIdx.x; rg < n_rg; rg += gridDim.x) {
    const int64_t gr = rg * tpb + team;
    if (gr >= nrows) continue;
    int64_t b, r;
    split_row(gr, A.rows, A.batch, b, r);
    const T *arow = act_tensor<T, Tab>(A.a, tab, b, E) + r * cols;
    T *prow = reinterpret_cast<T *>(A.payload + kHdrBytes + b * A.body_bytes) + r * cols;
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      if (v < V) {
        const typename Act<T>::Raw raw = Act<T>::load(arow + v * 8);
        float x[8];
        Act<T>::to_f32(raw, x);
        Act<T>::store_raw(prow + v * 8, raw);
        store_state8(reinterpret_cast<S *>(A.ahat) + gr * cols + v * 8, x);
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (A.err) store_state8(reinterpret_cast<S *>(A.err) + gr * cols + v * 8, z);
      }
    }
  }
}

// Step 0 receiver: ahat = fp32(body); recon = body.
template <typename T, int VPT, typename Tab, typename S = float>
__global__ void __launch_bounds__(kBlock) warm_decode_kernel(const DecArgs A, const __grid_constant__ Tab tab) {
  pdl_enter();
  if (!header_ok(A)) return;
  const int tlog = A.team_log2;
  const int TEAM = 1 << tlog;
  const int t = threadIdx.x & (TEAM - 1);
  const int team = threadIdx.x >> tlog;
  const int tpb = kBlock >> tlog;
  const int64_t cols = A.cols, E = A.rows * cols;
  const int V = (int)(cols >> 3);
  const int64_t nrows = (int64_t)A.batch * A.rows;
  const int64_t n_rg = (nrows + tpb - 1) / tpb;
  for (int64_t rg = blockIdx.x; rg < n_rg; rg += gridDim.x) {
    const int64_t gr = rg * tpb + team;
    if (gr >= nrows) continue;
    int64_t b, r;
    split_row(gr, A.rows, A.batch, b, r);
    const T *prow = reinterpret_cast<const T *>(A.payload + kHdrBytes + b * A.body_bytes) + r * cols;
    T *rrow = static_cast<T *>(recon_tensor<Tab>(A.recon, tab, b, E * (int64_t)sizeof(T))) + r * cols;
#pragma unroll
    for (int j = 0; j < VPT; j++) {
      const int v = t + (j << tlog);
      if (v < V) {
        const typename Act<T>::Raw raw = Act<T>::load(prow + v * 8);
        float x[8];
        Act<T>::to_f32(raw, x);
        store_state8(reinterpret_cast<S *>(A.ahat) + gr * cols + v * 8, x);
        Act<T>::store_raw(rrow + v * 8, raw);
      }
    }
  }
}

}  // namespace

// Kernel of one mode family (defined in cf_stream_mode_<mode>.cu).
const void *stream_kernel_id(bool enc, int dtype, int nm_m, int nm_n, int vpt, bool table, bool state_bf16);
const void *stream_kernel_s1(bool enc, int dtype, int nm_m, int nm_n, int vpt, bool table, bool state_bf16);
const void *stream_kernel_q2(bool enc, int dtype, int nm_m, int nm_n, int vpt, bool table, bool state_bf16);
const void *stream_kernel_nm(bool enc, int dtype, int nm_m, int nm_n, int vpt, bool table, bool state_bf16);

namespace {
template <int MODE, int NM_M, int NM_N, typename T, typename Tab, typename S, int VPT>
const void *pick_one(bool enc) {
  if (enc) return reinterpret_cast<const void *>(&encode_kernel<MODE, T, VPT, NM_M, NM_N, Tab, S>);
  return reinterpret_cast<const void *>(&decode_kernel<MODE, T, VPT, NM_M, NM_N, Tab, S>);
}

template <int MODE, int NM_M, int NM_N, typename T, typename Tab, typename S>
const void *pick(bool enc, int vpt) {
  switch (vpt) {
    case 1: return pick_one<MODE, NM_M, NM_N, T, Tab, S, 1>(enc);
    case 2: return pick_one<MODE, NM_M, NM_N, T, Tab, S, 2>(enc);
    case 3: return pick_one<MODE, NM_M, NM_N, T, Tab, S, 3>(enc);
    case 4: return pick_one<MODE, NM_M, NM_N, T, Tab, S, 4>(enc);
  }
  return nullptr;
}

// The bf16-state option exists for bf16 activations only.
template <int MODE, int NM_M, int NM_N>
const void *pick_any(bool enc, int dtype, int vpt, bool table, bool state_bf16) {
  if (dtype == CF_BF16) {
    if (state_bf16)
      return table ? pick<MODE, NM_M, NM_N, __nv_bfloat16, PtrTable, __nv_bfloat16>(enc, vpt)
                   : pick<MODE, NM_M, NM_N, __nv_bfloat16, NoTable, __nv_bfloat16>(enc, vpt);
    return table ? pick<MODE, NM_M, NM_N, __nv_bfloat16, PtrTable, float>(enc, vpt)
                 : pick<MODE, NM_M, NM_N, __nv_bfloat16, NoTable, float>(enc, vpt);
  }
  if (state_bf16) return nullptr;
  return table ? pick<MODE, NM_M, NM_N, float, PtrTable, float>(enc, vpt)
               : pick<MODE, NM_M, NM_N, float, NoTable, float>(enc, vpt);
}
}  // namespace

}  // namespace cfi
