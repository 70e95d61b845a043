// cf_api.cu -- host layer of libcf: the C ABI declared in include/cf.h.
//
// Owns the per-stream state (sender: ahat, e [, V_prev, low-rank scratch];
// receiver: ahat), validates every argument before any launch, builds the
// 64-byte payload header, and enqueues the fused kernels on the caller's
// stream.  No torch types, no exceptions across the ABI.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_set>

#include "cf.h"
#include "cf_blocksel.h"
#include "cf_internal.h"
#include "cf_lowrank.h"

using namespace cfi;

struct cf_state {
  int64_t rows = 0, cols = 0;
  int mode = 0;
  cf_params p{};
  int device = 0;
  int sm_count = 0;
  void *slab = nullptr;
  bool own_slab = false;
  size_t slab_bytes = 0;
  int *status = nullptr;
  float *ahat = nullptr;
  float *err = nullptr;
  float *vprev = nullptr;
  void *lr_scratch = nullptr;
  size_t lr_scratch_bytes = 0;
  uint64_t step = 0;
  StreamCfg cfg{};
  Layout lay{};
  LowrankPlan lr{};
  BlockselPlan bs{};
  // Low-rank sender: the encode chain (14 launches for one sweep) runs as
  // one CUDA graph, captured on a private stream at each call and swapped
  // into the executable graph with cudaGraphExecUpdate (same topology, new
  // arguments), so that the chain pays one graph launch instead of a stream
  // launch per kernel.
  cudaStream_t cap = nullptr;
  cudaGraphExec_t gexec = nullptr;
};

namespace {

std::mutex g_mu;
std::unordered_set<const cf_state *> g_live;

bool live(const cf_state *s) {
  std::lock_guard<std::mutex> lk(g_mu);
  return s && g_live.count(s);
}

size_t pad16(size_t b) { return (b + 15u) & ~(size_t)15u; }
size_t pad256(size_t b) { return (b + 255u) & ~(size_t)255u; }

int ilog2(int m) {
  int c = 0;
  while ((1 << c) < m) c++;
  return c;
}

size_t act_size(int dtype) { return dtype == CF_BF16 ? 2u : 4u; }

int bs_plan_of(int64_t rows, int64_t cols, const cf_params &p, BlockselPlan *P) {
  return blocksel_plan(rows, cols, p.dtype, p.batch, p.bs_grid_h, p.bs_block, p.bs_k, p.bs_warm, P);
}

Layout layout_of(int64_t rows, int64_t cols, int mode, const cf_params &p) {
  Layout L{};
  switch (mode) {
    case CF_IDENTITY:
      L.body = pad16((size_t)(rows * cols) * 4u);
      break;
    case CF_SIGN1:
      L.sec1 = pad16((size_t)rows * 2u);
      L.body = L.sec1 + pad16((size_t)(rows * cols / 8));
      break;
    case CF_Q2:
      L.sec1 = pad16((size_t)rows * 2u);
      L.body = L.sec1 + pad16((size_t)(rows * cols / 4));
      break;
    case CF_NM: {
      const int64_t blocks = cols / p.nm_m;
      const int64_t words = blocks * p.nm_n * ilog2(p.nm_m) / 32;
      L.sec1 = pad16((size_t)(rows * blocks * p.nm_n) * 2u);
      L.body = L.sec1 + pad16((size_t)(rows * words) * 4u);
      break;
    }
    case CF_BLOCKSEL: {
      BlockselPlan bp{};
      if (bs_plan_of(rows, cols, p, &bp) == CF_OK) {
        L.sec1 = pad16((size_t)bp.k * 4u);
        L.body = blocksel_body_bytes(bp);
      }
      break;
    }
    case CF_LOWRANK:
      if (p.lr_int4) {
        L.sec1 = pad16((size_t)p.rank * 8u);
        L.sec2 = L.sec1 + pad16((size_t)((rows * p.rank + 1) / 2));
        L.body = L.sec2 + pad16((size_t)((cols * p.rank + 1) / 2));
      } else {
        L.sec1 = 0;
        L.sec2 = pad16((size_t)(rows * p.rank) * 4u);
        L.body = L.sec2 + pad16((size_t)(cols * p.rank) * 4u);
      }
      break;
  }
  return L;
}

int validate(int64_t rows, int64_t cols, int mode, const cf_params *p) {
  if (!p) return CF_ERR_ARG;
  if (mode < CF_IDENTITY || mode > CF_BLOCKSEL) return CF_ERR_ARG;
  if (p->dtype != CF_F32 && p->dtype != CF_BF16) return CF_ERR_ARG;
  if (p->role != CF_SENDER && p->role != CF_RECEIVER) return CF_ERR_ARG;
  if (p->ef != CF_EF_EXPLICIT && p->ef != CF_EF_IMPLICIT && p->ef != CF_EF_OFF) return CF_ERR_ARG;
  if (p->batch < 1 || p->batch > kMaxBatch * 1024) return CF_ERR_ARG;
  if (rows < 1 || cols < 8) return CF_ERR_SHAPE;
  if (cols % 8) return CF_ERR_SHAPE;
  if (cols > kMaxCols) return CF_ERR_SHAPE;
  if (mode == CF_SIGN1 && cols % 32) return CF_ERR_SHAPE;
  if (mode == CF_Q2 && cols % 16) return CF_ERR_SHAPE;
  if (mode == CF_NM) {
    if (!((p->nm_m == 16 || p->nm_m == 4) && (p->nm_n == 1 || p->nm_n == 2) && p->nm_n < p->nm_m))
      return CF_ERR_UNSUPPORTED;
    if (cols % p->nm_m) return CF_ERR_SHAPE;
    if (((cols / p->nm_m) * p->nm_n * ilog2(p->nm_m)) % 32) return CF_ERR_SHAPE;
  }
  if (p->state_dtype != CF_F32 && p->state_dtype != CF_BF16) return CF_ERR_ARG;
  if (p->state_dtype == CF_BF16 && (p->dtype != CF_BF16 || mode == CF_LOWRANK || mode == CF_BLOCKSEL))
    return CF_ERR_UNSUPPORTED;  // the bf16 state is an option of the streaming modes on bf16 activations
  if (mode == CF_BLOCKSEL) {
    BlockselPlan bp{};
    const int rc = bs_plan_of(rows, cols, *p, &bp);
    if (rc != CF_OK) return rc;
  }
  if (mode == CF_LOWRANK) {
    if (p->rank < 1 || p->rank > kMaxRank || p->rank > rows || p->rank > cols) return CF_ERR_SHAPE;
    if (rows % 128 || cols % 128) return CF_ERR_SHAPE;
    if (p->iters < 1 || p->iters > 2) return CF_ERR_UNSUPPORTED;
    if (p->lr_int4 != 0 && p->lr_int4 != 1) return CF_ERR_ARG;
    if (!(p->lr_qr2_tol >= 0.0 && p->lr_qr2_tol <= 1.0 / 4096.0)) return CF_ERR_ARG;  // NaN fails too
    if (p->batch != 1) return CF_ERR_UNSUPPORTED;
    LowrankPlan plan{};
    lowrank_plan(rows, cols, *p, &plan);
    if (!plan.supported) return CF_ERR_UNSUPPORTED;
  }
  return CF_OK;
}

struct Carve {
  size_t status, ahat, err, vprev, lr, bs, total;
};

Carve carve_of(int64_t rows, int64_t cols, int mode, const cf_params &p, const LowrankPlan &lr,
               const BlockselPlan &bs) {
  Carve c{};
  const size_t E = (size_t)(rows * cols) * (size_t)p.batch;
  size_t off = 0;
  c.status = off;
  off += 256;
  const size_t esz = p.state_dtype == CF_BF16 ? 2u : 4u;
  c.ahat = off;
  off += pad256(E * esz);
  if (p.role == CF_SENDER && mode != CF_BLOCKSEL) {  // block selection keeps no error term
    c.err = off;
    off += pad256(E * esz);
    if (mode == CF_LOWRANK) {
      c.vprev = off;
      off += pad256((size_t)cols * p.rank * 4u * p.batch);
    }
  }
  if (mode == CF_LOWRANK) {
    c.lr = off;
    off += pad256(p.role == CF_SENDER ? lr.enc_scratch_bytes : lr.dec_scratch_bytes);
  }
  if (mode == CF_BLOCKSEL && p.role == CF_SENDER) {
    c.bs = off;
    off += pad256(blocksel_scratch_bytes(bs));
  }
  c.total = off;
  return c;
}

Header header_of(const cf_state *s, bool warm, uint64_t step) {
  Header h{};
  h.w[0] = kMagic;
  h.w[1] = (uint32_t)s->mode;
  h.w[2] = warm ? 1u : 0u;
  h.w[3] = (uint32_t)s->p.dtype;
  h.w[4] = (uint32_t)(step & 0xffffffffu);
  h.w[5] = (uint32_t)(step >> 32);
  h.w[6] = (uint32_t)((uint64_t)s->rows & 0xffffffffu);
  h.w[7] = (uint32_t)((uint64_t)s->rows >> 32);
  h.w[8] = (uint32_t)((uint64_t)s->cols & 0xffffffffu);
  h.w[9] = (uint32_t)((uint64_t)s->cols >> 32);
  h.w[10] = (uint32_t)s->p.batch;
  uint32_t p0 = 0, p1 = 0, p2 = 0;
  if (s->mode == CF_NM) { p0 = (uint32_t)s->p.nm_n; p1 = (uint32_t)s->p.nm_m; }
  if (s->mode == CF_LOWRANK) { p0 = (uint32_t)s->p.rank; p1 = (uint32_t)s->p.lr_int4; p2 = (uint32_t)s->p.iters; }
  if (s->mode == CF_BLOCKSEL) { p0 = (uint32_t)s->bs.H; p1 = (uint32_t)s->bs.b; p2 = (uint32_t)s->bs.k; }
  h.w[11] = p0;
  h.w[12] = p1;
  h.w[13] = (uint32_t)s->p.ef;
  h.w[14] = p2;
  h.w[15] = 0;
  return h;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int cuda_err(cudaError_t e) {
  if (e == cudaSuccess) return CF_OK;
  (void)cudaGetLastError();
  return CF_ERR_CUDA;
}

size_t warm_body(const cf_state *s) { return pad16((size_t)(s->rows * s->cols) * act_size(s->p.dtype)); }

// leading steps sent in full (block selection: bs_warm; every other mode: 1)
uint64_t warm_steps(const cf_state *s) { return s->mode == CF_BLOCKSEL ? (uint64_t)s->bs.warm : 1u; }

// bytes per element of the ahat tensor: fp32, except block selection, whose
// state holds raw activations in their own dtype
size_t ahat_elem_bytes(const cf_state *s) {
  if (s->mode == CF_BLOCKSEL) return act_size(s->p.dtype);
  return s->p.state_dtype == CF_BF16 ? 2u : 4u;
}

EncArgs enc_args(cf_state *s, const void *a, void *payload, bool warm) {
  EncArgs A{};
  A.a = a;
  A.ahat = s->ahat;
  A.err = s->err;
  A.payload = static_cast<uint8_t *>(payload);
  A.rows = s->rows;
  A.cols = s->cols;
  A.body_bytes = (int64_t)(warm ? warm_body(s) : s->lay.body);
  A.sec1 = (int64_t)s->lay.sec1;
  A.batch = s->p.batch;
  A.ef_explicit = s->p.ef == CF_EF_EXPLICIT;
  A.ef_off = s->p.ef == CF_EF_OFF;
  A.team_log2 = s->cfg.team_log2;
  A.status = s->status;
  A.hdr = header_of(s, warm, s->step);
  if (!warm) {
    // [end of first section, sec1) and [end of second section, body)
    size_t end1 = 0, end2 = 0;
    const int64_t R = s->rows, C = s->cols;
    switch (s->mode) {
      case CF_SIGN1: end1 = (size_t)R * 2u; end2 = s->lay.sec1 + (size_t)(R * C / 8); break;
      case CF_Q2: end1 = (size_t)R * 2u; end2 = s->lay.sec1 + (size_t)(R * C / 4); break;
      case CF_NM: {
        const int64_t blocks = C / s->p.nm_m;
        end1 = (size_t)(R * blocks * s->p.nm_n) * 2u;
        end2 = s->lay.sec1 + (size_t)(R * (blocks * s->p.nm_n * ilog2(s->p.nm_m) / 32)) * 4u;
        break;
      }
      default: end1 = s->lay.sec1; end2 = s->lay.body; break;
    }
    if (s->mode == CF_SIGN1 || s->mode == CF_Q2 || s->mode == CF_NM) {
      A.padA_off = (int64_t)end1;
      A.padA_len = (int64_t)(s->lay.sec1 - end1);
      A.padB_off = (int64_t)end2;
      A.padB_len = (int64_t)(s->lay.body - end2);
    }
  }
  return A;
}

DecArgs dec_args(cf_state *s, const void *payload, void *recon, bool warm) {
  DecArgs A{};
  A.payload = static_cast<const uint8_t *>(payload);
  A.recon = recon;
  A.ahat = s->ahat;
  A.status = s->status;
  A.rows = s->rows;
  A.cols = s->cols;
  A.body_bytes = (int64_t)(warm ? warm_body(s) : s->lay.body);
  A.sec1 = (int64_t)s->lay.sec1;
  A.batch = s->p.batch;
  A.team_log2 = s->cfg.team_log2;
  A.expect = header_of(s, warm, s->step);
  return A;
}

// Runs chain(stream) as a CUDA graph launched on st (see cf_state::gexec).
// When st is itself being captured, the launches go straight into the
// caller's graph.
template <typename F>
cudaError_t graph_run(cf_state *s, cudaStream_t st, F &&chain) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  if (cs != cudaStreamCaptureStatusNone) return chain(st);
  if (!s->cap && (e = cudaStreamCreateWithFlags(&s->cap, cudaStreamNonBlocking)) != cudaSuccess) {
    s->cap = nullptr;
    return e;
  }
  if ((e = cudaStreamBeginCapture(s->cap, cudaStreamCaptureModeThreadLocal)) != cudaSuccess) return e;
  const cudaError_t le = chain(s->cap);
  cudaGraph_t g = nullptr;
  e = cudaStreamEndCapture(s->cap, &g);
  if (le != cudaSuccess || e != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    (void)cudaGetLastError();
    return le != cudaSuccess ? le : e;
  }
  if (s->gexec) {
    cudaGraphExecUpdateResultInfo info{};
    if (cudaGraphExecUpdate(s->gexec, g, &info) != cudaSuccess) {  // topology changed: instantiate anew
      (void)cudaGetLastError();
      cudaGraphExecDestroy(s->gexec);
      s->gexec = nullptr;
    }
  }
  if (!s->gexec && (e = cudaGraphInstantiate(&s->gexec, g, 0)) != cudaSuccess) s->gexec = nullptr;
  cudaGraphDestroy(g);
  if (e != cudaSuccess) return e;
  return cudaGraphLaunch(s->gexec, st);
}

int do_encode(cf_state *s, const void *a, const PtrTable *tab, void *payload, cudaStream_t st) {
  if (!live(s)) return CF_ERR_STATE;
  if (s->p.role != CF_SENDER) return CF_ERR_ROLE;
  if (!payload || (!a && !tab)) return CF_ERR_ARG;
  if (!aligned16(payload) || (a && !aligned16(a))) return CF_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != s->device) return CF_ERR_ARG;
  const bool warm = s->step < warm_steps(s);
  if (s->mode == CF_BLOCKSEL && tab) return CF_ERR_UNSUPPORTED;
  EncArgs A = enc_args(s, a, payload, warm);
  cudaError_t e;
  if (s->mode == CF_BLOCKSEL) {
    e = blocksel_encode(s->bs, a, s->ahat, static_cast<uint8_t *>(payload), A.hdr, warm, st);
  } else if (warm) {
    e = launch_warm_encode(s->p.dtype, s->cfg, A, tab, st);
  } else if (s->mode == CF_LOWRANK) {
    e = graph_run(s, st, [&](cudaStream_t cs) { return lowrank_encode(s->lr, A, tab, s->vprev, s->step, s->p.seed, cs); });
  } else {
    e = launch_encode(s->mode, s->p.dtype, s->p.nm_m, s->p.nm_n, s->cfg, A, tab, st);
  }
  if (e != cudaSuccess) return cuda_err(e);
  s->step++;
  return CF_OK;
}

int do_decode(cf_state *s, const void *payload, void *recon, const PtrTable *tab, cudaStream_t st) {
  if (!live(s)) return CF_ERR_STATE;
  if (s->p.role != CF_RECEIVER) return CF_ERR_ROLE;
  if (!payload || (!recon && !tab)) return CF_ERR_ARG;
  if (!aligned16(payload) || (recon && !aligned16(recon))) return CF_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != s->device) return CF_ERR_ARG;
  const bool warm = s->step < warm_steps(s);
  if (s->mode == CF_BLOCKSEL && tab) return CF_ERR_UNSUPPORTED;
  DecArgs A = dec_args(s, payload, recon, warm);
  cudaError_t e;
  if (s->mode == CF_BLOCKSEL) {
    e = blocksel_decode(s->bs, static_cast<const uint8_t *>(payload), s->ahat, recon, A.expect, warm, s->status, st);
  } else if (warm) {
    e = launch_warm_decode(s->p.dtype, s->cfg, A, tab, st);
  } else if (s->mode == CF_LOWRANK) {
    e = lowrank_decode(s->lr, A, tab, st);  // two launches: a graph would not pay off
  } else {
    e = launch_decode(s->mode, s->p.dtype, s->p.nm_m, s->p.nm_n, s->cfg, A, tab, st);
  }
  if (e != cudaSuccess) return cuda_err(e);
  s->step++;
  return CF_OK;
}

int fill_table(const cf_state *s, const void *const *ptrs, PtrTable *tab) {
  if (!ptrs) return CF_ERR_ARG;
  if (s->p.batch > kMaxBatch) return CF_ERR_UNSUPPORTED;
  std::memset(tab, 0, sizeof(*tab));
  for (int b = 0; b < s->p.batch; b++) {
    if (!ptrs[b]) return CF_ERR_ARG;
    if (!aligned16(ptrs[b])) return CF_ERR_ALIGN;
    tab->p[b] = ptrs[b];
  }
  return CF_OK;
}

constexpr uint64_t kExportMagic = 0x3154534650434643ull;  // "CFCPFST1"

struct ExportHeader {
  uint64_t magic;
  int64_t rows, cols;
  int32_t mode, dtype, role, ef, nm_n, nm_m, rank, iters, lr_int4, batch;
  uint64_t step;
  int32_t status;
  int32_t state_dtype;
  uint64_t tensor_bytes;
};

}  // namespace

extern "C" {

const char *cf_version(void) { return "cf 0.1.0 (sm_100a)"; }

const char *cf_strerror(int status) {
  switch (status) {
    case CF_OK: return "ok";
    case CF_ERR_ARG: return "invalid argument";
    case CF_ERR_SHAPE: return "shape violates the mode's rules";
    case CF_ERR_ROLE: return "wrong role for this call (encode needs a sender, decode a receiver)";
    case CF_ERR_UNSUPPORTED: return "configuration not supported by this build";
    case CF_ERR_CUDA: return "CUDA runtime error";
    case CF_ERR_NOMEM: return "out of device memory or workspace too small";
    case CF_ERR_DESYNC: return "payload header did not match the receiver (mode, shape or step)";
    case CF_ERR_ALIGN: return "pointer not 16-byte aligned";
    case CF_ERR_STATE: return "not a live state";
    case CF_ERR_SIZE: return "host buffer size mismatch";
    case CF_ERR_TIMEOUT: return "a kernel's bounded wait for its own asynchronous copy gave up";
    case CF_ERR_TOO_LARGE: return "problem larger than the allocation-free entry point's fixed scratch";
  }
  return "unknown status";
}

int cf_params_init(cf_params *p) {
  if (!p) return CF_ERR_ARG;
  std::memset(p, 0, sizeof(*p));
  p->dtype = CF_BF16;
  p->role = CF_SENDER;
  p->ef = CF_EF_EXPLICIT;
  p->nm_n = 2;
  p->nm_m = 16;
  p->rank = 70;
  p->iters = 1;
  p->lr_int4 = 1;
  p->batch = 1;
  p->seed = 0;
  p->bs_grid_h = 0;
  p->bs_block = 8;
  p->bs_k = 0;
  p->bs_warm = 5;
  p->state_dtype = CF_F32;
  p->lr_qr2_tol = 1.0 / 65536.0;
  return CF_OK;
}

int cf_workspace_bytes(int64_t rows, int64_t cols, int mode, const cf_params *p, size_t *out) {
  if (!out) return CF_ERR_ARG;
  const int v = validate(rows, cols, mode, p);
  if (v != CF_OK) return v;
  LowrankPlan lr{};
  BlockselPlan bs{};
  if (mode == CF_LOWRANK) lowrank_plan(rows, cols, *p, &lr);
  if (mode == CF_BLOCKSEL) bs_plan_of(rows, cols, *p, &bs);
  *out = carve_of(rows, cols, mode, *p, lr, bs).total;
  return CF_OK;
}

int cf_create(int64_t rows, int64_t cols, int mode, const cf_params *p, cf_state **out) {
  if (!out) return CF_ERR_ARG;
  *out = nullptr;
  const int v = validate(rows, cols, mode, p);
  if (v != CF_OK) return v;
  cf_state *s = new (std::nothrow) cf_state();
  if (!s) return CF_ERR_NOMEM;
  s->rows = rows;
  s->cols = cols;
  s->mode = mode;
  s->p = *p;
  if (cudaGetDevice(&s->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&s->sm_count, cudaDevAttrMultiProcessorCount, s->device) != cudaSuccess) {
    (void)cudaGetLastError();
    delete s;
    return CF_ERR_CUDA;
  }
  if (mode == CF_LOWRANK) lowrank_plan(rows, cols, *p, &s->lr);
  if (mode == CF_BLOCKSEL) bs_plan_of(rows, cols, *p, &s->bs);
  s->lay = layout_of(rows, cols, mode, *p);
  const int rc = stream_config(mode, p->dtype, p->nm_m, p->nm_n, rows, cols, p->batch, s->sm_count,
                               p->state_dtype == CF_BF16, &s->cfg);
  if (rc != CF_OK) {
    delete s;
    return rc;
  }
  const Carve c = carve_of(rows, cols, mode, *p, s->lr, s->bs);
  if (p->workspace) {
    if (p->workspace_bytes < c.total || ((uintptr_t)p->workspace & 255u)) {
      delete s;
      return p->workspace_bytes < c.total ? CF_ERR_NOMEM : CF_ERR_ALIGN;
    }
    s->slab = p->workspace;
    s->own_slab = false;
  } else {
    if (cudaMalloc(&s->slab, c.total) != cudaSuccess) {
      (void)cudaGetLastError();
      delete s;
      return CF_ERR_NOMEM;
    }
    s->own_slab = true;
  }
  s->slab_bytes = c.total;
  uint8_t *base = static_cast<uint8_t *>(s->slab);
  s->status = reinterpret_cast<int *>(base + c.status);
  s->ahat = reinterpret_cast<float *>(base + c.ahat);
  s->err = (p->role == CF_SENDER && mode != CF_BLOCKSEL) ? reinterpret_cast<float *>(base + c.err) : nullptr;
  s->vprev = (p->role == CF_SENDER && mode == CF_LOWRANK) ? reinterpret_cast<float *>(base + c.vprev) : nullptr;
  s->lr_scratch = mode == CF_LOWRANK ? static_cast<void *>(base + c.lr) : nullptr;
  if (mode == CF_BLOCKSEL && p->role == CF_SENDER) {
    const int rc2 = blocksel_bind(&s->bs, base + c.bs);
    if (rc2 != CF_OK) {
      if (s->own_slab) cudaFree(s->slab);
      delete s;
      return rc2;
    }
  }
  if (mode == CF_LOWRANK) {
    const int rc2 = lowrank_bind(&s->lr, s->lr_scratch);
    if (rc2 != CF_OK) {
      if (s->own_slab) cudaFree(s->slab);
      delete s;
      return rc2;
    }
  }
  if (cudaMemsetAsync(s->slab, 0, c.total, 0) != cudaSuccess || cudaStreamSynchronize(0) != cudaSuccess) {
    (void)cudaGetLastError();
    if (s->own_slab) cudaFree(s->slab);
    delete s;
    return CF_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lk(g_mu);
    g_live.insert(s);
  }
  *out = s;
  return CF_OK;
}

int cf_payload_bytes(const cf_state *s, int warmup, size_t *out) {
  if (!live(s)) return CF_ERR_STATE;
  if (!out) return CF_ERR_ARG;
  const size_t body = warmup ? warm_body(s) : s->lay.body;
  *out = (size_t)kHdrBytes + body * (size_t)s->p.batch;
  return CF_OK;
}

int cf_encode(cf_state *s, const void *a, void *payload, void *stream) {
  if (!a) return CF_ERR_ARG;
  return do_encode(s, a, nullptr, payload, static_cast<cudaStream_t>(stream));
}

int cf_decode(cf_state *s, const void *payload, void *recon, void *stream) {
  if (!recon) return CF_ERR_ARG;
  return do_decode(s, payload, recon, nullptr, static_cast<cudaStream_t>(stream));
}

int cf_encode_batched(cf_state *s, const void *const *a_ptrs, void *payload, void *stream) {
  if (!live(s)) return CF_ERR_STATE;
  PtrTable *tab = new (std::nothrow) PtrTable;
  if (!tab) return CF_ERR_NOMEM;
  int rc = fill_table(s, a_ptrs, tab);
  if (rc == CF_OK) rc = do_encode(s, nullptr, tab, payload, static_cast<cudaStream_t>(stream));
  delete tab;
  return rc;
}

int cf_decode_batched(cf_state *s, const void *payload, void *const *recon_ptrs, void *stream) {
  if (!live(s)) return CF_ERR_STATE;
  PtrTable *tab = new (std::nothrow) PtrTable;
  if (!tab) return CF_ERR_NOMEM;
  int rc = fill_table(s, reinterpret_cast<const void *const *>(recon_ptrs), tab);
  if (rc == CF_OK) rc = do_decode(s, payload, nullptr, tab, static_cast<cudaStream_t>(stream));
  delete tab;
  return rc;
}

int cf_status(cf_state *s, void *stream) {
  if (!live(s)) return CF_ERR_STATE;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  int h = 0;
  if (cudaMemcpy(&h, s->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  if (h & 2) return CF_ERR_TIMEOUT;
  return (h & 1) ? CF_ERR_DESYNC : CF_OK;
}

int cf_tensor(cf_state *s, int which, void **dptr, size_t *bytes) {
  if (!live(s)) return CF_ERR_STATE;
  if (!dptr || !bytes) return CF_ERR_ARG;
  const size_t E = (size_t)(s->rows * s->cols) * (size_t)s->p.batch;
  switch (which) {
    case CF_T_RECON:
      *dptr = s->ahat;
      *bytes = E * ahat_elem_bytes(s);
      return CF_OK;
    case CF_T_ERROR:
      if (!s->err) return CF_ERR_ROLE;
      *dptr = s->err;
      *bytes = E * ahat_elem_bytes(s);
      return CF_OK;
    case CF_T_VPREV:
      if (!s->vprev) return CF_ERR_ROLE;
      *dptr = s->vprev;
      *bytes = (size_t)s->cols * s->p.rank * 4u * s->p.batch;
      return CF_OK;
  }
  return CF_ERR_ARG;
}

int cf_step(const cf_state *s, uint64_t *out) {
  if (!live(s)) return CF_ERR_STATE;
  if (!out) return CF_ERR_ARG;
  *out = s->step;
  return CF_OK;
}

int cf_reset(cf_state *s) {
  if (!live(s)) return CF_ERR_STATE;
  if (cudaMemsetAsync(s->slab, 0, s->slab_bytes, 0) != cudaSuccess || cudaStreamSynchronize(0) != cudaSuccess)
    return cuda_err(cudaErrorUnknown);
  s->step = 0;
  return CF_OK;
}

int cf_test_wait_timeout(cf_state *s, uint32_t polls) {
  if (!live(s)) return CF_ERR_STATE;
  if (s->mode != CF_LOWRANK) return CF_ERR_UNSUPPORTED;
  s->lr.test_wait_polls = polls;
  return CF_OK;
}

static size_t export_tensor_bytes(const cf_state *s) {
  const size_t E = (size_t)(s->rows * s->cols) * (size_t)s->p.batch;
  size_t b = E * ahat_elem_bytes(s);
  if (s->err) b += E * ahat_elem_bytes(s);
  if (s->vprev) b += (size_t)s->cols * s->p.rank * 4u * s->p.batch;
  if (s->bs.sent) b += (size_t)s->bs.K;
  return b;
}

int cf_state_bytes(const cf_state *s, size_t *out) {
  if (!live(s)) return CF_ERR_STATE;
  if (!out) return CF_ERR_ARG;
  *out = sizeof(ExportHeader) + export_tensor_bytes(s);
  return CF_OK;
}

int cf_state_export(const cf_state *s, void *host, size_t bytes, void *stream) {
  if (!live(s)) return CF_ERR_STATE;
  if (!host) return CF_ERR_ARG;
  if (bytes != sizeof(ExportHeader) + export_tensor_bytes(s)) return CF_ERR_SIZE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  ExportHeader h{};
  h.magic = kExportMagic;
  h.rows = s->rows; h.cols = s->cols; h.mode = s->mode; h.dtype = s->p.dtype; h.role = s->p.role;
  h.ef = s->p.ef; h.nm_n = s->p.nm_n; h.nm_m = s->p.nm_m; h.rank = s->p.rank; h.iters = s->p.iters;
  h.lr_int4 = s->p.lr_int4; h.batch = s->p.batch; h.step = s->step; h.state_dtype = s->p.state_dtype;
  h.tensor_bytes = export_tensor_bytes(s);
  if (cudaMemcpy(&h.status, s->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  uint8_t *dst = static_cast<uint8_t *>(host);
  std::memcpy(dst, &h, sizeof(h));
  dst += sizeof(h);
  const size_t E = (size_t)(s->rows * s->cols) * (size_t)s->p.batch;
  const size_t hb = E * ahat_elem_bytes(s);
  if (cudaMemcpy(dst, s->ahat, hb, cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  dst += hb;
  if (s->err) {
    if (cudaMemcpy(dst, s->err, hb, cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_err(cudaErrorUnknown);
    dst += hb;
  }
  if (s->vprev) {
    const size_t vb = (size_t)s->cols * s->p.rank * 4u * s->p.batch;
    if (cudaMemcpy(dst, s->vprev, vb, cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_err(cudaErrorUnknown);
    dst += vb;
  }
  if (s->bs.sent &&
      cudaMemcpy(dst, s->bs.sent, (size_t)s->bs.K, cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_err(cudaErrorUnknown);
  return CF_OK;
}

int cf_state_import(cf_state *s, const void *host, size_t bytes, void *stream) {
  if (!live(s)) return CF_ERR_STATE;
  if (!host) return CF_ERR_ARG;
  if (bytes != sizeof(ExportHeader) + export_tensor_bytes(s)) return CF_ERR_SIZE;
  ExportHeader h{};
  std::memcpy(&h, host, sizeof(h));
  if (h.magic != kExportMagic || h.rows != s->rows || h.cols != s->cols || h.mode != s->mode ||
      h.dtype != s->p.dtype || h.role != s->p.role || h.ef != s->p.ef || h.nm_n != s->p.nm_n ||
      h.nm_m != s->p.nm_m || h.rank != s->p.rank || h.iters != s->p.iters || h.lr_int4 != s->p.lr_int4 ||
      h.batch != s->p.batch || h.state_dtype != s->p.state_dtype || h.tensor_bytes != export_tensor_bytes(s))
    return CF_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  const uint8_t *src = static_cast<const uint8_t *>(host) + sizeof(h);
  const size_t E = (size_t)(s->rows * s->cols) * (size_t)s->p.batch;
  const size_t hb = E * ahat_elem_bytes(s);
  if (cudaMemcpy(s->ahat, src, hb, cudaMemcpyHostToDevice) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  src += hb;
  if (s->err) {
    if (cudaMemcpy(s->err, src, hb, cudaMemcpyHostToDevice) != cudaSuccess) return cuda_err(cudaErrorUnknown);
    src += hb;
  }
  if (s->vprev) {
    const size_t vb = (size_t)s->cols * s->p.rank * 4u * s->p.batch;
    if (cudaMemcpy(s->vprev, src, vb, cudaMemcpyHostToDevice) != cudaSuccess) return cuda_err(cudaErrorUnknown);
    src += vb;
  }
  if (s->bs.sent &&
      cudaMemcpy(s->bs.sent, src, (size_t)s->bs.K, cudaMemcpyHostToDevice) != cudaSuccess)
    return cuda_err(cudaErrorUnknown);
  if (cudaMemcpy(s->status, &h.status, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return cuda_err(cudaErrorUnknown);
  s->step = h.step;
  return CF_OK;
}

int cf_destroy(cf_state *s) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!s || !g_live.count(s)) return CF_ERR_STATE;
    g_live.erase(s);
  }
  cudaDeviceSynchronize();
  if (s->gexec) cudaGraphExecDestroy(s->gexec);
  if (s->cap) cudaStreamDestroy(s->cap);
  if (s->own_slab) cudaFree(s->slab);
  (void)cudaGetLastError();
  delete s;
  return CF_OK;
}

}  // extern "C"
