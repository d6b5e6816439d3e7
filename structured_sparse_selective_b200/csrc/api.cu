// C-ABI entry points of libpdssm.so: argument validation, workspace layout,
// device binding and dispatch. See include/pdssm.h for the contract.
#include <string.h>

#include <algorithm>
#include <mutex>

#include "launch.h"
#include "pdssm.h"

using namespace pdssm;

namespace {

size_t dtype_size(int dt) {
  switch (dt) {
    case PDSSM_F32: return 4;
    case PDSSM_BF16: return 2;
    case PDSSM_C64: return 8;
    default: return 0;
  }
}

bool mul_ok(int64_t a, int64_t b, int64_t *out) { return !__builtin_mul_overflow(a, b, out); }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Plan {
  int64_t Bt, L, H, N, P, K, T, nC, rows;
  int64_t Kd;         // dictionary entries: K, or heads * K with per-head dictionaries
  bool cplx;
  bool fused;         // the fused kernel serves the problem: the workspace is the error word only
  size_t state_size;  // bytes per state element (4 or 8)
  // workspace offsets
  size_t o_err, o_idx, o_off, o_src, o_s, o_cstate, o_cidx, o_cval, o_yloc, total;
};

int64_t default_chunk(const pdssm_problem *pb) {
  // Long enough that chunk-end states stay O(L*N) (T >= P) and the sequential
  // carry scan over chunks stays short; short enough that the chunk-parallel
  // phases still fill the GPU: about 1024 threads on each of the 148 SMs, in
  // blocks of 32 columns x the kernels' row groups (1, 2 or 8 by N).
  const int64_t col_blocks = (pb->P + 31) / 32;
  const int64_t row_groups = pb->N <= 16 ? 1 : (pb->N <= 32 ? 2 : 8);
  const int64_t want = 148 * 1024 / (32 * row_groups);
  int64_t T = 256;
  while (T > 64 && pb->batch * pb->heads * col_blocks * ((pb->seqlen + T - 1) / T) < want) T /= 2;
  return std::max<int64_t>(T, pb->P);
}

// Validates the problem and lays out its workspace. The layout follows the path
// the problem takes: the fused kernel (when it applies and `three_kernel` is
// false) needs only the error word; the three-kernel path needs the chunk
// states, pairs and local outputs as well.
pdssm_status make_plan(const pdssm_problem *pb, Plan *pl, bool three_kernel = false) {
  if (!pb) return PDSSM_ERR_INVALID_ARG;
  if (pb->batch < 0 || pb->seqlen < 0 || pb->heads < 0 || pb->N < 1 || pb->P < 1 || pb->K < 1 ||
      pb->chunk < 0)
    return PDSSM_ERR_INVALID_ARG;
  if (pb->N > PDSSM_MAX_N || pb->P > PDSSM_MAX_P || pb->K > PDSSM_MAX_K) return PDSSM_ERR_UNSUPPORTED;
  if (pb->batch > 65535 || pb->heads > 65535) return PDSSM_ERR_UNSUPPORTED;
  if (pb->logits_t != PDSSM_F32 && pb->logits_t != PDSSM_BF16) return PDSSM_ERR_UNSUPPORTED;
  if (pb->in_t != PDSSM_F32 && pb->in_t != PDSSM_BF16) return PDSSM_ERR_UNSUPPORTED;
  if (pb->state_t == PDSSM_F32) {
    if (pb->d_t != PDSSM_F32 && pb->d_t != PDSSM_BF16) return PDSSM_ERR_UNSUPPORTED;
    if (pb->out_t != PDSSM_F32 && pb->out_t != PDSSM_BF16) return PDSSM_ERR_UNSUPPORTED;
  } else if (pb->state_t == PDSSM_C64) {
    if (pb->d_t != PDSSM_C64 || pb->out_t != PDSSM_C64) return PDSSM_ERR_UNSUPPORTED;
  } else {
    return PDSSM_ERR_UNSUPPORTED;
  }
  if (pb->flags & ~(PDSSM_FLAG_DEVICE_CHECK | PDSSM_FLAG_REFERENCE_PATH | PDSSM_FLAG_SHORT_WAITS |
                    PDSSM_FLAG_HEAD_DICTS))
    return PDSSM_ERR_INVALID_ARG;

  Plan p;
  p.Bt = pb->batch; p.L = pb->seqlen; p.H = pb->heads; p.N = pb->N; p.P = pb->P; p.K = pb->K;
  p.cplx = pb->state_t == PDSSM_C64;
  p.state_size = p.cplx ? 8 : 4;
  p.T = pb->chunk ? pb->chunk : default_chunk(pb);
  p.nC = p.L > 0 ? (p.L + p.T - 1) / p.T : 0;
  int64_t bh, rows, tmp;
  if (!mul_ok(p.Bt, p.H, &bh) || !mul_ok(bh, p.L, &rows)) return PDSSM_ERR_UNSUPPORTED;
  if (!mul_ok(rows, std::max(std::max(p.N, p.P), p.K) * 8, &tmp)) return PDSSM_ERR_UNSUPPORTED;
  if (p.nC > INT32_MAX) return PDSSM_ERR_UNSUPPORTED;
  p.rows = rows;
  p.Kd = (pb->flags & PDSSM_FLAG_HEAD_DICTS) ? p.H * p.K : p.K;
  int64_t nchunks = bh * p.nC;
  p.fused = !three_kernel && fused_scan_applies(pb);
  size_t o = 0;
  p.o_err = o; o = align256(o + 4);
  if (p.fused) {
    p.o_idx = p.o_off = p.o_src = p.o_s = p.o_cstate = p.o_cidx = p.o_cval = p.o_yloc = o;
    p.total = o;
    *pl = p;
    return PDSSM_OK;
  }
  p.o_idx = o; o = align256(o + (size_t)(p.Kd * p.N) * 4);
  p.o_off = o; o = align256(o + (size_t)(p.Kd * (p.N + 1)) * 4);
  p.o_src = o; o = align256(o + (size_t)(p.Kd * p.N) * 4);
  p.o_s = o; o = align256(o + (size_t)rows * 4);
  p.o_cstate = o; o = align256(o + (size_t)nchunks * p.N * p.P * p.state_size);
  p.o_cidx = o; o = align256(o + (size_t)nchunks * p.N * 4);
  p.o_cval = o; o = align256(o + (size_t)nchunks * p.N * p.state_size);
  p.o_yloc = o; o = align256(o + (size_t)rows * p.P * p.state_size);
  p.total = o;
  *pl = p;
  return PDSSM_OK;
}

Workspace carve(const Plan &p, void *ws) {
  char *base = static_cast<char *>(ws);
  Workspace w;
  w.err = reinterpret_cast<uint32_t *>(base + p.o_err);
  w.idx = reinterpret_cast<int32_t *>(base + p.o_idx);
  w.csr_off = reinterpret_cast<int32_t *>(base + p.o_off);
  w.csr_src = reinterpret_cast<int32_t *>(base + p.o_src);
  w.s = reinterpret_cast<int32_t *>(base + p.o_s);
  w.chunk_state = base + p.o_cstate;
  w.chunk_idx = reinterpret_cast<int32_t *>(base + p.o_cidx);
  w.chunk_val = base + p.o_cval;
  w.y_loc = base + p.o_yloc;
  return w;
}

bool aligned(const void *ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

// Makes the device that owns `stream` current for this library's runtime.
pdssm_status bind_device(cudaStream_t stream) {
  if (stream == nullptr) return PDSSM_OK;
  int dev = -1;
  if (cudaStreamGetDevice(stream, &dev) != cudaSuccess) return PDSSM_ERR_CUDA;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return PDSSM_ERR_CUDA;
  if (cur != dev && cudaSetDevice(dev) != cudaSuccess) return PDSSM_ERR_CUDA;
  return PDSSM_OK;
}

pdssm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PDSSM_OK : PDSSM_ERR_CUDA; }

pdssm_status check_scan_args(const pdssm_problem *pb, const Plan &p, const int32_t *idx,
                             const void *d, const void *B, const void *C, const void *x,
                             const void *h0, const void *y, const void *h_final,
                             const int32_t *prod_idx, const void *prod_val, const void *ws,
                             size_t ws_bytes) {
  if (!idx) return PDSSM_ERR_INVALID_ARG;
  if (p.rows > 0 && (!d || !B || !C || !x || !y)) return PDSSM_ERR_INVALID_ARG;
  const size_t es_in = dtype_size(pb->in_t), es_d = dtype_size(pb->d_t), es_o = dtype_size(pb->out_t);
  if (!aligned(idx, 4) || !aligned(d, es_d) || !aligned(B, es_in) || !aligned(C, es_in) ||
      !aligned(x, es_in) || !aligned(y, es_o) || !aligned(h0, p.state_size) ||
      !aligned(h_final, p.state_size) || !aligned(prod_idx, 4) || !aligned(prod_val, p.state_size))
    return PDSSM_ERR_INVALID_ARG;
  if (!ws || ws_bytes < p.total) return PDSSM_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return PDSSM_ERR_INVALID_ARG;
  return PDSSM_OK;
}

pdssm_status finish(const pdssm_problem *pb, const Workspace &w, cudaStream_t stream) {
  if (cudaGetLastError() != cudaSuccess) return PDSSM_ERR_CUDA;
  if (pb->flags & PDSSM_FLAG_DEVICE_CHECK) return pdssm_read_device_check(w.err, stream);
  return PDSSM_OK;
}

pdssm_status run_scan(const pdssm_problem *pb, const Plan &plan, const int32_t *s,
                      const void *logits, int32_t *s_out, const int32_t *idx, const void *d,
                      const void *B, const void *C, const void *x, const void *h0, void *y,
                      void *h_final, int32_t *prod_idx, void *prod_val, void *workspace,
                      size_t workspace_bytes, cudaStream_t stream, const uint8_t *steps = nullptr) {
  Plan p = plan;
  ScanArgs a;
  a.s = s; a.logits = logits; a.d = d; a.B = B; a.C = C; a.x = x; a.steps = steps;
  if (steps && (!p.fused || !fused_scan_pointers_ok(a))) return PDSSM_ERR_UNSUPPORTED;
  if (p.fused && !fused_scan_pointers_ok(a)) {
    // inputs the fused kernel's 16-byte loads cannot read: the three-kernel
    // path runs instead and needs its own (larger) workspace
    pdssm_status st = make_plan(pb, &p, true);
    if (st != PDSSM_OK) return st;
    if (workspace_bytes < p.total) return PDSSM_ERR_WORKSPACE;
  }
  Workspace w = carve(p, workspace);
  if (cudaMemsetAsync(w.err, 0, 4, stream) != cudaSuccess) return PDSSM_ERR_CUDA;
  pdssm_status st = PDSSM_OK;

  a.Bt = p.Bt; a.L = p.L; a.H = p.H; a.N = p.N; a.P = p.P; a.K = p.K; a.T = p.T; a.nC = p.nC;
  a.d_t = pb->d_t; a.in_t = pb->in_t; a.out_t = pb->out_t; a.logits_t = pb->logits_t;
  a.cplx = p.cplx;
  a.s = s; a.logits = logits; a.s_out = s_out; a.idx = idx; a.steps = steps;
  a.d = d; a.B = B; a.C = C; a.x = x; a.h0 = h0; a.y = y; a.h_final = h_final;
  a.prod_idx = prod_idx; a.prod_val = prod_val; a.ws = w;
  a.short_waits = (pb->flags & PDSSM_FLAG_SHORT_WAITS) != 0;
  a.head_dicts = (pb->flags & PDSSM_FLAG_HEAD_DICTS) != 0;

  if (p.Bt * p.H == 0) return finish(pb, w, stream);
  if (p.L == 0) {
    st = cuda_status(launch_empty_outputs(a, stream));
    return st != PDSSM_OK ? st : finish(pb, w, stream);
  }
  if (p.fused) {
    // the fused kernel validates idx itself and needs no preimage lists
    st = cuda_status(launch_fused_scan(a, stream));
    return st != PDSSM_OK ? st : finish(pb, w, stream);
  }
  st = cuda_status(launch_prep_dict(idx, (int)p.Kd, (int)p.N, w, stream));
  if (st != PDSSM_OK) return st;
  if (!a.s) {
    // unfused selection into s_out (or the workspace)
    int32_t *sbuf = s_out ? s_out : w.s;
    st = cuda_status(launch_select(pb->logits_t, logits, p.rows, (int)p.K, sbuf, stream));
    if (st != PDSSM_OK) return st;
    a.s = sbuf;
  }
  st = cuda_status(launch_chunked_scan(a, stream));
  if (st != PDSSM_OK) return st;
  return finish(pb, w, stream);
}

// Workspace of the backward pass: error word, dictionary preimage lists,
// checkpoints [Bt][H][nCk][N][P] and the per-slice scratch [Bt][H][16][N][P].
struct BwdPlan {
  int64_t Bt, L, H, N, P, K, rows, nCk, Kd, state_size, nPB;
  size_t o_err, o_idx, o_off, o_src, o_ckpt, o_cidx, o_cval, o_scr, o_pdd, o_pdB, o_pdC, o_pdpi, total;
};

pdssm_status make_bwd_plan(const pdssm_problem *pb, BwdPlan *bp) {
  Plan p;
  pdssm_status st = make_plan(pb, &p, true);
  if (st != PDSSM_OK) return st;
  BwdPlan q;
  q.nPB = scan_bwd_column_blocks(p.Bt * p.H, p.P, p.cplx);
  // more column blocks (narrower blocks) until one block's shared memory fits
  while (scan_bwd_smem_bytes(p.N, p.P / q.nPB, p.K, p.cplx) > (size_t)227 * 1024 && p.P % (2 * q.nPB) == 0)
    q.nPB *= 2;
  if (scan_bwd_smem_bytes(p.N, p.P / q.nPB, p.K, p.cplx) > (size_t)227 * 1024) return PDSSM_ERR_UNSUPPORTED;
  q.state_size = p.state_size;
  q.Bt = p.Bt; q.L = p.L; q.H = p.H; q.N = p.N; q.P = p.P; q.K = p.K; q.rows = p.rows; q.Kd = p.Kd;
  q.nCk = scan_bwd_checkpoints(p.L);
  int64_t slices = p.Bt * p.H, per_slice, tot;
  if (!mul_ok(p.N * p.P, q.nCk + scan_bwd_scratch_steps(), &per_slice) || !mul_ok(slices, per_slice, &tot) ||
      !mul_ok(tot, p.state_size, &tot))
    return PDSSM_ERR_UNSUPPORTED;
  size_t o = 0;
  q.o_err = o; o = align256(o + 4);
  q.o_idx = o; o = align256(o + (size_t)(p.Kd * p.N) * 4);
  q.o_off = o; o = align256(o + (size_t)(p.Kd * (p.N + 1)) * 4);
  q.o_src = o; o = align256(o + (size_t)(p.Kd * p.N) * 4);
  // checkpoints: the chunked forward's carries at chunk length 16, with its chunk pairs
  q.o_ckpt = o; o = align256(o + (size_t)(slices * q.nCk * p.N * p.P) * p.state_size);
  q.o_cidx = o; o = align256(o + (size_t)(slices * q.nCk * p.N) * 4);
  q.o_cval = o; o = align256(o + (size_t)(slices * q.nCk * p.N) * p.state_size);
  q.o_scr = o; o = align256(o + (size_t)(slices * scan_bwd_scratch_steps() * p.N * p.P) * p.state_size);
  // the column blocks' shares of the sums over columns (none with one block a sequence)
  int64_t parts64 = 0, check;
  if (q.nPB > 1 && (!mul_ok(q.nPB, p.rows, &parts64) || !mul_ok(parts64, (p.N + p.K) * 16, &check)))
    return PDSSM_ERR_UNSUPPORTED;
  const size_t parts = (size_t)parts64;
  q.o_pdd = o; o = align256(o + parts * p.N * p.state_size);
  q.o_pdB = o; o = align256(o + parts * p.N * 4);
  q.o_pdC = o; o = align256(o + parts * p.N * 4);
  q.o_pdpi = o; o = align256(o + parts * p.K * 4);
  q.total = o;
  *bp = q;
  return PDSSM_OK;
}

constexpr int kMaxTraced = 64;
struct TraceState {
  void *const *events = nullptr;
  int32_t n_events = 0;
  int32_t used = 0;
  bool on = false;
  const char *names[kMaxTraced] = {};
};
thread_local TraceState g_trace;

}  // namespace

namespace pdssm {

cudaError_t trace_before(cudaStream_t st, const char *kernel_name) {
  TraceState &t = g_trace;
  if (!t.on || 2 * (t.used + 1) > t.n_events || t.used >= kMaxTraced) return cudaSuccess;
  t.names[t.used] = kernel_name;
  return cudaEventRecord(static_cast<cudaEvent_t>(t.events[2 * t.used]), st);
}

cudaError_t trace_after(cudaStream_t st) {
  TraceState &t = g_trace;
  if (!t.on || 2 * (t.used + 1) > t.n_events || t.used >= kMaxTraced) return cudaSuccess;
  cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(t.events[2 * t.used + 1]), st);
  ++t.used;
  return e;
}

}  // namespace pdssm

extern "C" {

pdssm_status pdssm_trace_begin(void *const *events, int32_t n_events) {
  if (n_events < 0 || (n_events > 0 && !events)) return PDSSM_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n_events; ++i)
    if (!events[i]) return PDSSM_ERR_INVALID_ARG;
  g_trace.events = events;
  g_trace.n_events = n_events;
  g_trace.used = 0;
  g_trace.on = true;
  for (int i = 0; i < kMaxTraced; ++i) g_trace.names[i] = nullptr;
  return PDSSM_OK;
}

int32_t pdssm_trace_end(void) {
  g_trace.on = false;
  g_trace.events = nullptr;
  g_trace.n_events = 0;
  return g_trace.used;
}

const char *pdssm_trace_kernel_name(int32_t i) {
  if (i < 0 || i >= g_trace.used || i >= kMaxTraced) return nullptr;
  return g_trace.names[i];
}


const char *pdssm_status_string(int32_t status) {
  switch (status) {
    case PDSSM_OK: return "PDSSM_OK";
    case PDSSM_ERR_INVALID_ARG: return "PDSSM_ERR_INVALID_ARG: invalid argument";
    case PDSSM_ERR_UNSUPPORTED: return "PDSSM_ERR_UNSUPPORTED: size or dtype combination not supported";
    case PDSSM_ERR_WORKSPACE: return "PDSSM_ERR_WORKSPACE: workspace missing or too small";
    case PDSSM_ERR_CUDA: return "PDSSM_ERR_CUDA: CUDA launch or runtime error";
    case PDSSM_ERR_DEVICE_CHECK: return "PDSSM_ERR_DEVICE_CHECK: idx or s value out of range";
    case PDSSM_ERR_TIMEOUT: return "PDSSM_ERR_TIMEOUT: bounded device wait gave up";
    default: return "PDSSM_ERR_UNKNOWN";
  }
}

const char *pdssm_version(void) { return "0.1.0"; }

pdssm_status pdssm_workspace_size(const pdssm_problem *pb, size_t *bytes) {
  if (!bytes) return PDSSM_ERR_INVALID_ARG;
  Plan p;
  pdssm_status st = make_plan(pb, &p);
  if (st != PDSSM_OK) return st;
  *bytes = p.total;
  return PDSSM_OK;
}

pdssm_status pdssm_select(const pdssm_problem *pb, const void *logits, int32_t *s,
                          pdssm_stream_t stream) {
  Plan p;
  pdssm_status st = make_plan(pb, &p);
  if (st != PDSSM_OK) return st;
  if (p.rows == 0) return PDSSM_OK;
  if (!logits || !s) return PDSSM_ERR_INVALID_ARG;
  if (!aligned(logits, dtype_size(pb->logits_t)) || !aligned(s, 4)) return PDSSM_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = bind_device(cs)) != PDSSM_OK) return st;
  return cuda_status(launch_select(pb->logits_t, logits, p.rows, (int)p.K, s, cs));
}

pdssm_status pdssm_scan_fwd(const pdssm_problem *pb, const int32_t *s, const int32_t *idx,
                            const void *d, const void *B, const void *C, const void *x,
                            const void *h0, void *y, void *h_final, int32_t *prod_idx,
                            void *prod_val, void *workspace, size_t workspace_bytes,
                            pdssm_stream_t stream) {
  Plan p;
  pdssm_status st = make_plan(pb, &p);
  if (st != PDSSM_OK) return st;
  if (p.rows > 0 && (!s || !aligned(s, 4))) return PDSSM_ERR_INVALID_ARG;
  st = check_scan_args(pb, p, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val, workspace,
                       workspace_bytes);
  if (st != PDSSM_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = bind_device(cs)) != PDSSM_OK) return st;
  return run_scan(pb, p, s, nullptr, nullptr, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val,
                  workspace, workspace_bytes, cs);
}

pdssm_status pdssm_forward(const pdssm_problem *pb, const void *logits, const int32_t *idx,
                           const void *d, const void *B, const void *C, const void *x,
                           const void *h0, void *y, void *h_final, int32_t *prod_idx,
                           void *prod_val, int32_t *s_out, void *workspace,
                           size_t workspace_bytes, pdssm_stream_t stream) {
  Plan p;
  pdssm_status st = make_plan(pb, &p);
  if (st != PDSSM_OK) return st;
  if (p.rows > 0 && (!logits || !aligned(logits, dtype_size(pb->logits_t)))) return PDSSM_ERR_INVALID_ARG;
  if (!aligned(s_out, 4)) return PDSSM_ERR_INVALID_ARG;
  st = check_scan_args(pb, p, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val, workspace,
                       workspace_bytes);
  if (st != PDSSM_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = bind_device(cs)) != PDSSM_OK) return st;
  return run_scan(pb, p, nullptr, logits, s_out, idx, d, B, C, x, h0, y, h_final, prod_idx,
                  prod_val, workspace, workspace_bytes, cs);
}

pdssm_status pdssm_dict_hardmax(int64_t K, int64_t N, const float *M, int32_t *idx, pdssm_stream_t stream) {
  if (K < 0 || N < 1) return PDSSM_ERR_INVALID_ARG;
  if (N > PDSSM_MAX_N) return PDSSM_ERR_UNSUPPORTED;
  if (K == 0) return PDSSM_OK;
  if (!M || !idx || !aligned(M, 4) || !aligned(idx, 4)) return PDSSM_ERR_INVALID_ARG;
  int64_t kn;
  if (!mul_ok(K, N * N, &kn)) return PDSSM_ERR_UNSUPPORTED;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  pdssm_status st = bind_device(cs);
  if (st != PDSSM_OK) return st;
  return cuda_status(launch_dict_hardmax(K, (int)N, M, idx, cs));
}

pdssm_status pdssm_select_proj(const pdssm_problem *pb, int64_t D, const void *u, const void *W, int32_t *s,
                               float *logits, void *workspace, size_t workspace_bytes, pdssm_stream_t stream) {
  if (!pb || pb->batch < 0 || pb->seqlen < 0 || pb->heads < 1 || pb->K < 1 || D < 1) return PDSSM_ERR_INVALID_ARG;
  if (pb->K > PDSSM_MAX_K || pb->heads > 65535 || !proj_select_supported(D, pb->heads, pb->K))
    return PDSSM_ERR_UNSUPPORTED;
  int64_t rows;
  if (!mul_ok(pb->batch, pb->seqlen, &rows)) return PDSSM_ERR_UNSUPPORTED;
  if (rows > 0 && (!u || !W || !s)) return PDSSM_ERR_INVALID_ARG;
  if (!aligned(u, 16) || !aligned(W, 16) || !aligned(s, 4) || !aligned(logits, 16)) return PDSSM_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < 256) return PDSSM_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return PDSSM_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  pdssm_status st = bind_device(cs);
  if (st != PDSSM_OK) return st;
  uint32_t *err = static_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(err, 0, 4, cs) != cudaSuccess) return PDSSM_ERR_CUDA;
  if (rows == 0) return PDSSM_OK;
  return cuda_status(launch_proj_select(rows, D, pb->heads, pb->K, u, W, s, logits, err, cs));
}

pdssm_status pdssm_soft_select_workspace_size(const pdssm_problem *pb, size_t *bytes) {
  if (!bytes) return PDSSM_ERR_INVALID_ARG;
  Plan p;
  pdssm_status st = make_plan(pb, &p, true);
  if (st != PDSSM_OK) return st;
  if (!soft_select_supported(p.N, p.K)) return PDSSM_ERR_UNSUPPORTED;
  *bytes = 256 + soft_select_ws_bytes((pb->flags & PDSSM_FLAG_HEAD_DICTS) ? p.H : 1, p.N, p.K);
  return PDSSM_OK;
}

pdssm_status pdssm_soft_select(const pdssm_problem *pb, const void *logits, const float *M, float tau,
                               uint8_t *idx_steps, void *workspace, size_t workspace_bytes,
                               pdssm_stream_t stream) {
  size_t need = 0;
  pdssm_status st = pdssm_soft_select_workspace_size(pb, &need);
  if (st != PDSSM_OK) return st;
  if (!(tau > 0.f) || !(tau < INFINITY)) return PDSSM_ERR_INVALID_ARG;
  Plan p;
  make_plan(pb, &p, true);
  if (p.rows > 0 && (!logits || !M || !idx_steps)) return PDSSM_ERR_INVALID_ARG;
  if (!aligned(logits, dtype_size(pb->logits_t)) || !aligned(M, 4)) return PDSSM_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < need) return PDSSM_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return PDSSM_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = bind_device(cs)) != PDSSM_OK) return st;
  uint32_t *err = static_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(err, 0, 4, cs) != cudaSuccess) return PDSSM_ERR_CUDA;
  if (p.rows == 0) return PDSSM_OK;
  return cuda_status(launch_soft_select(p.Bt * p.L, p.H, p.N, p.K, pb->logits_t, logits, M,
                                        (pb->flags & PDSSM_FLAG_HEAD_DICTS) != 0, tau,
                                        static_cast<char *>(workspace) + 256, idx_steps, err, cs));
}

pdssm_status pdssm_scan_fwd_steps(const pdssm_problem *pb, const uint8_t *idx_steps, const void *d, const void *B,
                                  const void *C, const void *x, const void *h0, void *y, void *h_final,
                                  int32_t *prod_idx, void *prod_val, void *workspace, size_t workspace_bytes,
                                  pdssm_stream_t stream) {
  if (!pb) return PDSSM_ERR_INVALID_ARG;
  // there are no logits and no dictionary: K and logits_t are not used
  pdssm_problem q = *pb;
  q.K = 16;
  q.logits_t = PDSSM_BF16;
  q.flags &= ~PDSSM_FLAG_HEAD_DICTS;
  pb = &q;
  Plan p;
  pdssm_status st = make_plan(pb, &p);
  if (st != PDSSM_OK) return st;
  if (!p.fused) return PDSSM_ERR_UNSUPPORTED;
  if (p.rows > 0 && (!idx_steps || !aligned(idx_steps, 16))) return PDSSM_ERR_INVALID_ARG;
  // the dictionary argument of the shared checks is unused here
  st = check_scan_args(pb, p, reinterpret_cast<const int32_t *>(idx_steps ? (const void *)idx_steps : d), d, B, C,
                       x, h0, y, h_final, prod_idx, prod_val, workspace, workspace_bytes);
  if (st != PDSSM_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = bind_device(cs)) != PDSSM_OK) return st;
  return run_scan(pb, p, nullptr, nullptr, nullptr, nullptr, d, B, C, x, h0, y, h_final, prod_idx, prod_val,
                  workspace, workspace_bytes, cs, idx_steps);
}

pdssm_status pdssm_bwd_workspace_size(const pdssm_problem *pb, size_t *bytes) {
  if (!bytes) return PDSSM_ERR_INVALID_ARG;
  BwdPlan q;
  pdssm_status st = make_bwd_plan(pb, &q);
  if (st != PDSSM_OK) return st;
  *bytes = q.total;
  return PDSSM_OK;
}

pdssm_status pdssm_scan_bwd(const pdssm_problem *pb, const void *logits, const int32_t *s,
                            const int32_t *idx, const void *d, const void *B, const void *C,
                            const void *x, const void *h0, const void *dy, const void *dh_final,
                            float tau, float *dlogits, void *dd, float *dB, float *dC, float *dx,
                            void *dh0, void *workspace, size_t workspace_bytes,
                            pdssm_stream_t stream) {
  BwdPlan q;
  pdssm_status st = make_bwd_plan(pb, &q);
  if (st != PDSSM_OK) return st;
  if (!idx || !(tau > 0.f) || !(tau < INFINITY)) return PDSSM_ERR_INVALID_ARG;
  if ((logits == nullptr) != (dlogits == nullptr)) return PDSSM_ERR_INVALID_ARG;
  if (q.rows > 0 && (!s || !d || !B || !C || !x || !dy || !dd || !dB || !dC || !dx))
    return PDSSM_ERR_INVALID_ARG;
  const size_t es_in = dtype_size(pb->in_t), es_d = dtype_size(pb->d_t), es_o = dtype_size(pb->out_t);
  const size_t es_s = (size_t)q.state_size;
  if (!aligned(idx, 4) || !aligned(s, 4) || !aligned(d, es_d) || !aligned(B, es_in) || !aligned(C, es_in) ||
      !aligned(x, es_in) || !aligned(dy, es_o) || !aligned(logits, dtype_size(pb->logits_t)) ||
      !aligned(h0, es_s) || !aligned(dh_final, es_s) || !aligned(dlogits, 4) || !aligned(dd, es_s) ||
      !aligned(dB, 4) || !aligned(dC, 4) || !aligned(dx, 4) || !aligned(dh0, es_s))
    return PDSSM_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < q.total) return PDSSM_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return PDSSM_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = bind_device(cs)) != PDSSM_OK) return st;

  char *base = static_cast<char *>(workspace);
  Workspace w{};
  w.err = reinterpret_cast<uint32_t *>(base + q.o_err);
  w.idx = reinterpret_cast<int32_t *>(base + q.o_idx);
  w.csr_off = reinterpret_cast<int32_t *>(base + q.o_off);
  w.csr_src = reinterpret_cast<int32_t *>(base + q.o_src);
  if (cudaMemsetAsync(w.err, 0, 4, cs) != cudaSuccess) return PDSSM_ERR_CUDA;
  const int64_t slices = q.Bt * q.H;
  if (slices == 0) return finish(pb, w, cs);
  if (q.L == 0) {  // no steps: the final state is the initial one
    if (dh0) {
      const size_t n = (size_t)(slices * q.N * q.P) * es_s;
      cudaError_t e = dh_final ? cudaMemcpyAsync(dh0, dh_final, n, cudaMemcpyDeviceToDevice, cs)
                               : cudaMemsetAsync(dh0, 0, n, cs);
      if (e != cudaSuccess) return PDSSM_ERR_CUDA;
    }
    return finish(pb, w, cs);
  }
  st = cuda_status(launch_prep_dict(idx, (int)q.Kd, (int)q.N, w, cs));
  if (st != PDSSM_OK) return st;
  {
    // the checkpoints: the states after each 16-step chunk, by phases A and B of the
    // chunked forward scan (parallel over the chunks)
    ScanArgs f{};
    f.Bt = q.Bt; f.L = q.L; f.H = q.H; f.N = q.N; f.P = q.P; f.K = q.K;
    f.T = scan_bwd_scratch_steps(); f.nC = q.nCk;
    f.d_t = pb->d_t; f.in_t = pb->in_t; f.out_t = pb->out_t; f.logits_t = pb->logits_t;
    f.cplx = q.state_size == 8;
    f.s = s; f.idx = idx; f.d = d; f.B = B; f.C = C; f.x = x; f.h0 = h0;
    f.ws = w;
    f.ws.chunk_state = base + q.o_ckpt;
    f.ws.chunk_idx = reinterpret_cast<int32_t *>(base + q.o_cidx);
    f.ws.chunk_val = base + q.o_cval;
    f.head_dicts = (pb->flags & PDSSM_FLAG_HEAD_DICTS) != 0;
    st = cuda_status(launch_chunked_carries(f, cs));
    if (st != PDSSM_OK) return st;
  }
  ScanBwdArgs a;
  a.head_dicts = (pb->flags & PDSSM_FLAG_HEAD_DICTS) != 0;
  a.Bt = q.Bt; a.L = q.L; a.H = q.H; a.N = q.N; a.P = q.P; a.K = q.K;
  a.d_t = pb->d_t; a.in_t = pb->in_t; a.out_t = pb->out_t; a.logits_t = pb->logits_t;
  a.tau = tau;
  a.s = s; a.logits = logits; a.d = d; a.B = B; a.C = C; a.x = x; a.dy = dy;
  a.h0 = h0; a.dh_final = dh_final;
  a.ckpt = base + q.o_ckpt;
  a.scratch = base + q.o_scr;
  a.nPB = q.nPB;
  if (q.nPB > 1) {
    a.pdd = base + q.o_pdd;
    a.pdB = reinterpret_cast<float *>(base + q.o_pdB);
    a.pdC = reinterpret_cast<float *>(base + q.o_pdC);
    a.pdpi = reinterpret_cast<float *>(base + q.o_pdpi);
  }
  a.dlogits = dlogits; a.dd = dd; a.dB = dB; a.dC = dC; a.dx = dx; a.dh0 = dh0;
  a.ws = w;
  st = cuda_status(launch_scan_bwd(a, cs));
  if (st != PDSSM_OK) return st;
  return finish(pb, w, cs);
}

pdssm_status pdssm_read_device_check(const void *workspace, pdssm_stream_t stream) {
  if (!workspace) return PDSSM_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  pdssm_status st = bind_device(cs);
  if (st != PDSSM_OK) return st;
  uint32_t word = 0;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return PDSSM_ERR_CUDA;
  if (cudaMemcpy(&word, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return PDSSM_ERR_CUDA;
  if (word & kErrTimeout) return PDSSM_ERR_TIMEOUT;
  if (word & (kErrIdxRange | kErrSRange)) return PDSSM_ERR_DEVICE_CHECK;
  return PDSSM_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------
// Allocation-free variant of pdssm_forward.
//
// Some callers cannot call cudaMalloc on their call path: plug-ins whose host
// application already owns all device memory (a framework's caching
// allocator has reserved it), and latency-critical loops where cudaMalloc's
// implicit device synchronisation is not acceptable. For them the workspace
// lives in a fixed-size array in this library's device image instead of a
// caller buffer. Every GPU that loads the library holds the array until the
// process exits. All calls on a device share it, and it keeps the last call's
// contents; calls that overlap on the GPU (different streams, or different
// threads without ordering) race on it.

namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_static_ws_mutex;
void *g_static_ws_ptr[kMaxDevices] = {};

// Device address of the static workspace on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with that device current and cached. Only a successful lookup is cached: a
// call that fails (for instance inside a stream capture, where the lookup may
// be refused) returns PDSSM_ERR_CUDA and the next call tries again.
pdssm_status static_workspace(void **ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PDSSM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (!g_static_ws_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) {
      cudaGetLastError();  // the failure is reported by status; leave no sticky runtime error behind
      return PDSSM_ERR_CUDA;
    }
    g_static_ws_ptr[dev] = p;
  }
  *ptr = g_static_ws_ptr[dev];
  return PDSSM_OK;
}

}  // namespace

extern "C" pdssm_status pdssm_forward_noalloc(const pdssm_problem *pb, const void *logits,
                                              const int32_t *idx, const void *d, const void *B,
                                              const void *C, const void *x, const void *h0, void *y,
                                              void *h_final, int32_t *prod_idx, void *prod_val,
                                              int32_t *s_out, pdssm_stream_t stream) {
  Plan p;
  pdssm_status st = make_plan(pb, &p);
  if (st != PDSSM_OK) return st;
  if (p.total > kStaticWorkspaceBytes) return PDSSM_ERR_WORKSPACE;
  if (p.rows > 0 && (!logits || !aligned(logits, dtype_size(pb->logits_t)))) return PDSSM_ERR_INVALID_ARG;
  if (!aligned(s_out, 4)) return PDSSM_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((st = bind_device(cs)) != PDSSM_OK) return st;
  void *ws = nullptr;
  if ((st = static_workspace(&ws)) != PDSSM_OK) return st;
  st = check_scan_args(pb, p, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val, ws,
                       kStaticWorkspaceBytes);
  if (st != PDSSM_OK) return st;
  return run_scan(pb, p, nullptr, logits, s_out, idx, d, B, C, x, h0, y, h_final, prod_idx,
                  prod_val, ws, kStaticWorkspaceBytes, cs);
}
