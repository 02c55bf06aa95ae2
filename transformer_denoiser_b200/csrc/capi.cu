// C ABI of the two-stage DDIM denoiser (declared in include/kimodo.h).
//
// Host-side orchestration only: argument checks, device memory of the weights and
// the activation workspace, the order of kernel launches for one network forward
// ("Kimodo WebGPU", "Model details": 16 post-norm encoder layers), the two-stage
// step ("Architecture" figure: root -> globalRootToLocalRoot -> body -> CFG ->
// DDIM) and the CUDA graph that holds the whole sampling loop.  Every arithmetic
// step of the path runs in the kernels of this directory; the host computes only
// constants (the sinusoid table, the noise schedule and the per-step DDIM
// coefficients, in double precision).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/kimodo.h"
#include "../../include/kimodo_kernels.h"
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

using namespace kd;

namespace {

thread_local std::string g_last_error;

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define KD_CUDA(call)                                                                              \
  do {                                                                                             \
    cudaError_t e_ = (call);                                                                       \
    if (e_ != cudaSuccess)                                                                         \
      return set_error(e_ == cudaErrorMemoryAllocation ? KIMODO_ENOMEM : KIMODO_ECUDA, "%s: %s (%s:%d)", \
                       #call, cudaGetErrorString(e_), __FILE__, __LINE__);                         \
  } while (0)

#define KD_TRY(call)        \
  do {                      \
    int s_ = (call);        \
    if (s_ != KIMODO_OK) return s_; \
  } while (0)

#ifndef KD_SAMPLE_GROUPS
#define KD_SAMPLE_GROUPS 2
#endif
constexpr int SAMPLE_GROUPS = KD_SAMPLE_GROUPS;
// a call is split into prompt groups only when each group keeps at least this many token
// rows per network forward: measured, 64 ragged prompts (about 11,600 rows per group) run 8 %
// faster in two groups, 16 prompts of 150 frames (2,416 rows per group) 11 % slower
constexpr int GROUP_MIN_ROWS = 8192;

enum LaunchClass { CLS_GEMM_TC = 0, CLS_ATTN = 1, CLS_LN = 2, CLS_MOTION = 3, CLS_GEMM_F32 = 4, CLS_SETUP = 5,
                   NUM_CLS = 8 };

struct NetW {
  void* txt_W = nullptr; void* t_W1 = nullptr; void* t_W2 = nullptr; void* in_W = nullptr; void* out_W = nullptr;
  void* qkv_W[L] = {}; void* o_W[L] = {}; void* ff1_W[L] = {}; void* ff2_W[L] = {};
  float* txt_b = nullptr; float* t_b1 = nullptr; float* t_b2 = nullptr; float* in_b = nullptr; float* out_b = nullptr;
  float* qkv_b[L] = {}; float* o_b[L] = {}; float* ln1_g[L] = {}; float* ln1_b[L] = {};
  float* ff1_b[L] = {}; float* ff2_b[L] = {}; float* ln2_g[L] = {}; float* ln2_b[L] = {};
  int din = 0, dout = 0, in_ld = 0;
};

struct Workspace {
  int cap_rows = 0, cap_seq = 0, cap_frames = 0, cap_steps = 0;
  void* arena = nullptr;
  void* h = nullptr; void* qkv = nullptr; void* attn = nullptr; void* u = nullptr; float* y = nullptr;
  void* A_root = nullptr; void* A_body = nullptr;
  float* root_hat = nullptr; float* body_hat = nullptr; float* x = nullptr;
  void* emb = nullptr; float* txt[2] = {}; void* tpe = nullptr; void* thid = nullptr; float* tmlp[2] = {};
  int* lengths = nullptr; float* st_text = nullptr; float* st_null = nullptr;
  int* tok0 = nullptr; int* row_seq = nullptr;   // packed token layout (valid tokens only)
  float* stats[2] = {};                           // LayerNorm row statistics (mean, 1/std) [M][2]
};

// Token rows of a call: the padded layout (every sequence frames + 1 rows) or, when the
// lengths are known on the host and some sequence is shorter than `frames`, the packed
// layout of the valid tokens only (sequence s owns rows tok0[s] .. tok0[s + 1] - 1).
struct Tokens {
  int M = 0;
  bool packed = false;
};

struct ProfRec {
  cudaEvent_t a, b;
  int cls;
  double flops, bytes;
};

}  // namespace

struct kimodo_ctx {
  int device = 0;
  int precision = KIMODO_BF16;
  int num_sms = 148;
  void* warena = nullptr;
  NetW net[2];
  float* pe = nullptr;          // [N_TRAIN, D] sinusoid table (positions and timesteps)
  DevError* derr = nullptr;
  double alphabar[2][N_TRAIN];   // [KIMODO_SCHEDULE_LINEAR / _COSINE][t]
  Workspace ws;
  cudaStream_t cap_stream = nullptr;
  // sampler graphs keyed by (batch, frames, steps, null broadcast | takes << 1, cfg bits, schedule, eta bits, step noise,
  // token rows: the packed layout's row count, or the padded one)
  std::map<std::tuple<int, int, int, int, uint32_t, int, uint32_t, const float*, int>,
           std::pair<cudaGraphExec_t, long long>>
      graphs;
  float* zbuf = nullptr;        // staging of host step-noise draws
  size_t zcap = 0;              // floats
  bool profiling = false;
  unsigned prof_flags = cudaEventRecordDefault;   // cudaEventRecordExternal while a profiled graph is captured
  std::vector<ProfRec> prof;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
  long long launches = 0;
  long long last_launches = 0;
  Tokens tk;                    // token layout of the call being enqueued
  // Prompt groups of the sampler: the prompts of a large call are split into
  // SAMPLE_GROUPS halves whose whole sampling loops run as independent branches of the
  // graph (own workspace, own stream), so that one group's kernels fill the SMs the
  // other's leave idle (tails of the GEMMs, attention, LayerNorm).
  Workspace gws[SAMPLE_GROUPS];
  cudaStream_t gst[SAMPLE_GROUPS] = {};
  cudaEvent_t gev[SAMPLE_GROUPS + 1] = {};
  bool bf16() const { return precision == KIMODO_BF16; }
  size_t elem() const { return bf16() ? 2 : 4; }
};

namespace {

// ------------------------------------------------------------------ launch bookkeeping

cudaEvent_t next_event(kimodo_ctx* c) {
  if (c->ev_used == c->ev_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    c->ev_pool.push_back(e);
  }
  return c->ev_pool[c->ev_used++];
}

template <class Fn>
int launch(kimodo_ctx* c, int cls, double flops, double bytes, cudaStream_t st, const char* what, Fn fn) {
  ++c->launches;
  cudaEvent_t a = nullptr, b = nullptr;
  if (c->profiling) {
    a = next_event(c);
    b = next_event(c);
    if (a && b) cudaEventRecordWithFlags(a, st, c->prof_flags);
  }
  cudaError_t e = fn();
  if (e != cudaSuccess) return set_error(KIMODO_ECUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  if (c->profiling && a && b) {
    cudaEventRecordWithFlags(b, st, c->prof_flags);
    c->prof.push_back({a, b, cls, flops, bytes});
  }
  return KIMODO_OK;
}

// Token rows from which the layer projections run on the CTA-pair kernel.
constexpr int PAIR_GEMM_MIN_ROWS = 1024;

int pick_bn(const kimodo_ctx* c, int M, int N, int kind, bool out_f32) {
  if (N <= 16) return 16;
  if (N < 1024) return 128;
  // A few hundred tokens: every tile streams its full K extent of A and B, so the time is
  // set by the bytes one SM loads; the narrowest tile whose grid still fits in one wave
  // spreads the weights over the most SMs (the column split leaves each output
  // element's summation order unchanged).
  const bool narrow = (!out_f32 && (kind == EPI_BIAS || kind == EPI_BIAS_GELU)) ||
                      (out_f32 && (kind == EPI_BIAS_RESID || kind == EPI_BIAS_RESID_LN));
  if (narrow) {
    const long mt = (M + 127) / 128;
    for (int bn : {32, 64, 128})
      if (mt * ((N + bn - 1) / bn) <= c->num_sms) return bn;
  }
  auto eff = [&](int bn) {
    const long tiles = (long)((M + 127) / 128) * ((N + bn - 1) / bn);
    const long waves = (tiles + c->num_sms - 1) / c->num_sms;
    return (double)tiles / (double)(waves * c->num_sms);
  };
  return eff(256) + 1e-9 >= eff(128) ? 256 : 128;
}

// One projection: out = epilogue(A[M,K] . W[N,K]^T).
int gemm(kimodo_ctx* c, const void* A, int lda, const void* W, int ldw, int M, int N, int K, int kind,
         bool out_f32, const EpiParams& ep, cudaStream_t st, int cls_override = -1) {
  GemmArgs g;
  g.A = A; g.B = W; g.M = M; g.N = N; g.K = K; g.lda = lda; g.ldb = ldw;
  const double flops = 2.0 * M * N * K;
  const double bytes = (double)c->elem() * ((double)M * K + (double)N * K) +
                       (double)M * N * (out_f32 ? 4.0 : (double)c->elem()) +
                       (kind == EPI_BIAS_RESID || kind == EPI_BIAS_RESID_LN ? (double)M * N * 4.0 : 0.0);
  if (c->bf16()) {
    if (M >= PAIR_GEMM_MIN_ROWS && N >= 256 && gemm_tc2_supports(kind, out_f32)) {
      const int bn = gemm_tc2_pick_bn(M, N, kind);
      return launch(c, cls_override >= 0 ? cls_override : CLS_GEMM_TC, flops, bytes, st, "gemm_tc2",
                    [&] { return gemm_tc2(g, bn, kind, out_f32, ep, c->derr, st); });
    }
    const int bn = pick_bn(c, M, N, kind, out_f32);
    return launch(c, cls_override >= 0 ? cls_override : CLS_GEMM_TC, flops, bytes, st, "gemm_tc",
                  [&] { return gemm_tc(g, bn, kind, out_f32, ep, c->derr, st, c->num_sms); });
  }
  return launch(c, cls_override >= 0 ? cls_override : CLS_GEMM_F32, flops, bytes, st, "gemm_f32",
                [&] { return gemm_f32(g, kind, ep, st); });
}

// ------------------------------------------------------------------ weights

__global__ void convert_matrix_kernel(const float* __restrict__ src, int rows, int cols, void* dst, int ld,
                                      int to_bf16) {
  const long total = (long)rows * ld;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int r = i / ld, col = i % ld;
    const float v = col < cols ? src[(long)r * cols + col] : 0.f;
    if (to_bf16)
      static_cast<bf16*>(dst)[i] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(dst)[i] = v;
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Walks the canonical blob order; in "plan" mode only sizes the arena.
struct WeightWalker {
  kimodo_ctx* c;
  const float* src;     // device copy of the blob (nullptr while planning)
  size_t src_off = 0;
  char* arena;          // nullptr while planning
  size_t arena_off = 0;
  cudaStream_t st;
  int err = 0;

  void* matrix(int rows, int cols, int ld) {
    const size_t bytes = align256((size_t)rows * ld * c->elem());
    void* dst = arena ? arena + arena_off : nullptr;
    if (arena && !err) {
      const long total = (long)rows * ld;
      int grid = (int)((total + 255) / 256);
      grid = grid > 148 * 32 ? 148 * 32 : grid;
      convert_matrix_kernel<<<grid, 256, 0, st>>>(src + src_off, rows, cols, dst, ld, c->bf16() ? 1 : 0);
      if (cudaGetLastError() != cudaSuccess) err = 1;
    }
    arena_off += bytes;
    src_off += (size_t)rows * cols;
    return dst;
  }
  float* vec(int n) {
    const size_t bytes = align256((size_t)n * 4);
    float* dst = arena ? reinterpret_cast<float*>(arena + arena_off) : nullptr;
    if (arena && !err && cudaMemcpyAsync(dst, src + src_off, (size_t)n * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      err = 1;
    arena_off += bytes;
    src_off += n;
    return dst;
  }
  void net(NetW& n, int din, int dout, int in_ld) {
    n.din = din; n.dout = dout; n.in_ld = in_ld;
    n.txt_W = matrix(D, DTXT, DTXT); n.txt_b = vec(D);
    n.t_W1 = matrix(D, D, D); n.t_b1 = vec(D);
    n.t_W2 = matrix(D, D, D); n.t_b2 = vec(D);
    n.in_W = matrix(D, din, in_ld); n.in_b = vec(D);
    for (int l = 0; l < L; ++l) {
      n.qkv_W[l] = matrix(3 * D, D, D); n.qkv_b[l] = vec(3 * D);
      n.o_W[l] = matrix(D, D, D); n.o_b[l] = vec(D);
      n.ln1_g[l] = vec(D);
      n.ln1_b[l] = vec(D);
      n.ff1_W[l] = matrix(F, D, D); n.ff1_b[l] = vec(F);
      n.ff2_W[l] = matrix(D, F, F); n.ff2_b[l] = vec(D);
      n.ln2_g[l] = vec(D);
      n.ln2_b[l] = vec(D);
    }
    n.out_W = matrix(dout, D, D); n.out_b = vec(dout);
  }
  void all() {
    net(c->net[0], ROOT_F, ROOT_F, ROOT_IN_LD);
    net(c->net[1], MOTION_F, BODY_F, BODY_IN_LD);
  }
};

// ------------------------------------------------------------------ workspace

void free_graphs(kimodo_ctx* c) {
  for (auto& kv : c->graphs) cudaGraphExecDestroy(kv.second.first);
  c->graphs.clear();
}

// Grows workspace w to hold nseq sequences of `frames` frames and `steps` timestep rows;
// *grown tells whether it was (re)allocated, which invalidates graphs captured on it.
int alloc_workspace(kimodo_ctx* c, Workspace& w, int nseq, int frames, int steps, bool* grown) {
  const int S = frames + 1;
  const int rows = nseq * S;
  *grown = false;
  if (w.arena && rows <= w.cap_rows && nseq <= w.cap_seq && frames <= w.cap_frames && steps <= w.cap_steps)
    return KIMODO_OK;
  *grown = true;
  const int R = rows > w.cap_rows ? rows : w.cap_rows;
  const int NS = nseq > w.cap_seq ? nseq : w.cap_seq;
  const int TF = frames > w.cap_frames ? frames : w.cap_frames;
  const int ST = steps > w.cap_steps ? steps : w.cap_steps;
  const int R2 = NS * (TF + 1) > R ? NS * (TF + 1) : R;
  if (w.arena) cudaFree(w.arena);
  w = Workspace();
  const size_t e = c->elem();
  size_t off = 0;
  std::vector<std::pair<void**, size_t>> plan = {
      {&w.h, (size_t)R2 * D * e},          {&w.qkv, (size_t)R2 * 3 * D * e},
      {&w.attn, (size_t)R2 * D * e},       {&w.u, (size_t)R2 * F * e},
      {(void**)&w.y, (size_t)R2 * D * 4},  {&w.A_root, (size_t)R2 * ROOT_IN_LD * e},
      {&w.A_body, (size_t)R2 * BODY_IN_LD * e},
      {(void**)&w.root_hat, (size_t)NS * TF * ROOT_F * 4}, {(void**)&w.body_hat, (size_t)NS * TF * BODY_F * 4},
      {(void**)&w.x, (size_t)NS * TF * MOTION_F * 4},      {&w.emb, (size_t)NS * DTXT * e},
      {(void**)&w.txt[0], (size_t)NS * D * 4},             {(void**)&w.txt[1], (size_t)NS * D * 4},
      {&w.tpe, (size_t)ST * D * e},                        {&w.thid, (size_t)ST * D * e},
      {(void**)&w.tmlp[0], (size_t)ST * D * 4},            {(void**)&w.tmlp[1], (size_t)ST * D * 4},
      {(void**)&w.lengths, (size_t)NS * 4},                {(void**)&w.st_text, (size_t)NS * DTXT * 4},
      {(void**)&w.st_null, (size_t)NS * DTXT * 4},        {(void**)&w.tok0, (size_t)(NS + 1) * 4},
      {(void**)&w.row_seq, (size_t)R2 * 4},               {(void**)&w.stats[0], (size_t)R2 * 8},
      {(void**)&w.stats[1], (size_t)R2 * 8}};
  for (auto& p : plan) off += align256(p.second);
  void* arena = nullptr;
  cudaError_t err = cudaMalloc(&arena, off);
  if (err != cudaSuccess) {
    cudaGetLastError();
    return set_error(KIMODO_ENOMEM, "workspace allocation of %zu bytes failed: %s", off, cudaGetErrorString(err));
  }
  // zero once: the padded K columns of the input matrices must read as 0
  KD_CUDA(cudaMemset(arena, 0, off));
  w.arena = arena;
  off = 0;
  for (auto& p : plan) {
    *p.first = static_cast<char*>(arena) + off;
    off += align256(p.second);
  }
  w.cap_rows = R2; w.cap_seq = NS; w.cap_frames = TF; w.cap_steps = ST;
  return KIMODO_OK;
}

int ensure_workspace(kimodo_ctx* c, int nseq, int frames, int steps) {
  bool grown = false;
  const int r = alloc_workspace(c, c->ws, nseq, frames, steps, &grown);
  if (grown) free_graphs(c);
  return r;
}

// ------------------------------------------------------------------ forward pieces

// Sinusoid rows of the n_t timesteps t0, t0 - stride, ... (shared by both networks).
// Sinusoid rows of the n_t timesteps of this call: one explicit t (steps == 0) or the
// trailing timesteps of a `steps`-step sampler.
int timestep_rows(kimodo_ctx* c, int t_single, int steps, int n_t, cudaStream_t st) {
  return launch(c, CLS_SETUP, 0, (double)n_t * D * 8, st, "gather_timestep_rows",
                [&] { return gather_timestep_rows(c->pe, t_single, steps, n_t, c->ws.tpe, c->bf16(), st); });
}

// k-th trailing timestep of a `steps`-step sampler: floor(1000 (steps - k) / steps + 1/2) - 1
// (-1 for k == steps).
int trailing_t(int k, int steps) { return (2 * N_TRAIN * (steps - k) + steps) / (2 * steps) - 1; }

// Condition vectors of one network: text projection of the packed embeddings
// (rows) and the timestep MLP of the n_t gathered timestep rows.
int condition_setup(kimodo_ctx* c, int net, int rows, int n_t, cudaStream_t st) {
  NetW& n = c->net[net];
  Workspace& w = c->ws;
  EpiParams e;
  e.bias = n.txt_b; e.out = w.txt[net]; e.ldo = D; e.N = D; e.M = rows;
  KD_TRY(gemm(c, w.emb, DTXT, n.txt_W, DTXT, rows, D, DTXT, EPI_BIAS, true, e, st, CLS_SETUP));
  EpiParams e1;
  e1.bias = n.t_b1; e1.out = w.thid; e1.ldo = D; e1.N = D; e1.M = n_t;
  KD_TRY(gemm(c, w.tpe, D, n.t_W1, D, n_t, D, D, EPI_BIAS_SILU, !c->bf16(), e1, st, CLS_SETUP));
  EpiParams e2;
  e2.bias = n.t_b2; e2.out = w.tmlp[net]; e2.ldo = D; e2.N = D; e2.M = n_t;
  KD_TRY(gemm(c, w.thid, D, n.t_W2, D, n_t, D, D, EPI_BIAS, true, e2, st, CLS_SETUP));
  return KIMODO_OK;
}

// One network forward over nseq sequences of S = T + 1 tokens.  A_in holds the
// frame features (rows seq*S + 1 + i), tvec the timestep-MLP row of this call,
// txt the per-sequence text projection.  Output [nseq, T, dout] fp32 into hat.
int run_net(kimodo_ctx* c, int net, int nseq, int T, int len_mod, const void* A_in, const float* tvec,
            const float* txt, float* hat, cudaStream_t st) {
  NetW& n = c->net[net];
  Workspace& w = c->ws;
  const int S = T + 1;
  const bool packed = c->tk.packed;
  const int M = packed ? c->tk.M : nseq * S;
  const int* tok0 = packed ? w.tok0 : nullptr;
  const int* row_seq = packed ? w.row_seq : nullptr;
  const bool act_f32 = !c->bf16();
  {
    EpiParams e;
    e.bias = n.in_b; e.out = w.h; e.ldo = D; e.pe = c->pe; e.cond = txt; e.tvec = tvec; e.S = S; e.N = D; e.M = M;
    e.tok0 = tok0; e.row_seq = row_seq;
    if (c->bf16()) e.out32 = w.y;   // fp32 residual stream
    KD_TRY(gemm(c, A_in, n.in_ld, n.in_W, n.in_ld, M, D, n.in_ld, EPI_INPROJ, act_f32, e, st));
  }
  // Residual stream.  The residual epilogues write the sub-layer sums z into the fp32
  // buffer y.  bf16 path: y also serves as the residual, holding the un-normalised sums;
  // LayerNorm writes only the bf16 GEMM operand h and (mean, 1/std) per row, and the
  // next residual epilogue adds gamma (z - mean) / std + beta itself (EPI_BIAS_RESID_LN).
  // fp32 path: LayerNorm writes the normalised fp32 rows into h, which is the residual.
  const bool bf = c->bf16();
  const void* resid = bf ? static_cast<const void*>(w.y) : w.h;
  const double eb = (double)c->elem();
  auto resid_epi = [&](EpiParams& e, int which, const float* g, const float* b) {
    if (!bf || g == nullptr) return EPI_BIAS_RESID;
    e.ln_stats = w.stats[which];
    e.ln_g = g;
    e.ln_b = b;
    return EPI_BIAS_RESID_LN;
  };
  // Weights of the projections ahead, pulled into L2 by the kernels between them when the
  // projections run on the single-CTA kernel (below 1024 tokens, where a projection's
  // weights would otherwise come from HBM inside its K loop; the CTA-pair kernel pulls
  // its own weights into L2 before its dependency wait, and there the extra prefetch
  // slowed attention): attention fetches the rest of its layer (attention output, FFN1,
  // FFN2), the second LayerNorm the next layer's QKV weights.  A layer's weights are
  // consecutive in the arena (QKV, attention output, LayerNorm 1, FFN1, FFN2, LayerNorm 2).
  const bool prefetch_ahead = bf && M < PAIR_GEMM_MIN_ROWS;
  auto span = [prefetch_ahead](const void* a, const void* b) {
    L2Prefetch p;
    const uintptr_t ua = reinterpret_cast<uintptr_t>(a), ub = reinterpret_cast<uintptr_t>(b);
    if (prefetch_ahead && a != nullptr && ub > ua && (ua & 15) == 0 && ((ub - ua) & 15) == 0) {
      p.p = a;
      p.bytes = ub - ua;
    }
    return p;
  };
  for (int l = 0; l < L; ++l) {
    const L2Prefetch pf_layer = span(n.o_W[l], l + 1 < L ? n.qkv_W[l + 1] : n.out_W);
    const L2Prefetch pf_next = l + 1 < L ? span(n.qkv_W[l + 1], n.o_W[l + 1]) : L2Prefetch{};
    EpiParams e;
    e.bias = n.qkv_b[l]; e.out = w.qkv; e.ldo = 3 * D; e.N = 3 * D; e.M = M;
    KD_TRY(gemm(c, w.h, D, n.qkv_W[l], D, M, 3 * D, D, EPI_BIAS, act_f32, e, st));
    const double aflops = packed ? 4.0 * (double)M * S * DH * H : 4.0 * (double)nseq * S * S * DH * H;
    const double abytes = (double)M * 3 * D * eb + (double)M * D * eb;
    if (bf) {
      KD_TRY(launch(c, CLS_ATTN, aflops, abytes, st, "attention_tc", [&] {
        return attention_tc(static_cast<const bf16*>(w.qkv), static_cast<bf16*>(w.attn), M, w.lengths, len_mod,
                            nseq, S, c->derr, st, tok0, pf_layer);
      }));
    } else {
      KD_TRY(launch(c, CLS_ATTN, aflops, abytes, st, "attention_f32", [&] {
        return attention_f32(static_cast<const float*>(w.qkv), static_cast<float*>(w.attn), w.lengths, len_mod,
                             nseq, S, st, tok0);
      }));
    }
    EpiParams eo;
    eo.bias = n.o_b[l]; eo.out = w.y; eo.ldo = D; eo.resid = resid; eo.ldr = D;
    eo.N = D; eo.M = M;
    // layer 0 adds the un-normalised input projection; later layers the previous LayerNorm 2
    const int ko = resid_epi(eo, 1, l > 0 ? n.ln2_g[l - 1] : nullptr, l > 0 ? n.ln2_b[l - 1] : nullptr);
    KD_TRY(gemm(c, w.attn, D, n.o_W[l], D, M, D, D, ko, true, eo, st));
    const double lnb = bf ? (double)M * D * (4.0 + eb) + (double)M * 8 : (double)M * D * 8.0;
    KD_TRY(launch(c, CLS_LN, 0, lnb, st, "layernorm", [&] {
      return layernorm(w.y, w.h, bf, n.ln1_g[l], n.ln1_b[l], M, st, bf ? w.stats[0] : nullptr);
    }));
    EpiParams e1;
    e1.bias = n.ff1_b[l]; e1.out = w.u; e1.ldo = F; e1.N = F; e1.M = M;
    KD_TRY(gemm(c, w.h, D, n.ff1_W[l], D, M, F, D, EPI_BIAS_GELU, act_f32, e1, st));
    EpiParams e2;
    e2.bias = n.ff2_b[l]; e2.out = w.y; e2.ldo = D; e2.resid = resid; e2.ldr = D;
    e2.N = D; e2.M = M;
    const int kf = resid_epi(e2, 0, n.ln1_g[l], n.ln1_b[l]);
    KD_TRY(gemm(c, w.u, F, n.ff2_W[l], F, M, D, F, kf, true, e2, st));
    KD_TRY(launch(c, CLS_LN, 0, lnb, st, "layernorm", [&] {
      return layernorm(w.y, w.h, bf, n.ln2_g[l], n.ln2_b[l], M, st, bf ? w.stats[1] : nullptr, pf_next);
    }));
  }
  EpiParams eo;
  eo.bias = n.out_b; eo.out = hat; eo.ldo = n.dout; eo.lengths = w.lengths; eo.len_mod = len_mod; eo.S = S;
  eo.T = T; eo.N = n.dout; eo.M = M; eo.tok0 = tok0; eo.row_seq = row_seq;
  return gemm(c, w.h, D, n.out_W, D, M, n.dout, D, EPI_OUTPROJ, true, eo, st);
}

// DDIM update coefficients (double on the host):
//   sigma = eta sqrt((1 - ap) / (1 - at)) sqrt(1 - at / ap),
//   x_prev = sqrt(ap) x0 + sqrt(1 - ap - sigma^2) (x_t - sqrt(at) x0) / sqrt(1 - at) + sigma z
//          = c0 x0 + c1 x_t + c2 z.
void ddim_coeffs(const kimodo_ctx* c, int schedule, int t, int t_prev, double eta, float* c0, float* c1,
                 float* c2) {
  const double at = c->alphabar[schedule][t];
  const double ap = t_prev < 0 ? 1.0 : c->alphabar[schedule][t_prev];
  const double sigma = eta * sqrt((1.0 - ap) / (1.0 - at)) * sqrt(1.0 - at / ap);
  const double k1 = sqrt(fmax(1.0 - ap - sigma * sigma, 0.0)) / sqrt(1.0 - at);
  *c0 = (float)(sqrt(ap) - k1 * sqrt(at));
  *c1 = (float)k1;
  *c2 = (float)sigma;
}

// Sampler options after validation.
struct Sampler {
  int schedule = KIMODO_SCHEDULE_LINEAR;
  float eta = 0.f;
  const float* z = nullptr;   // device draws for the call (eta > 0), step-major
  int takes = 1;              // sequences per text-embedding row (variations of one prompt)
};

// One two-stage step for B prompts (cond rows 0..B-1, uncond rows B..2B-1).
// Reads ws.x, writes ws.x.  tvec_root / tvec_body are the timestep-MLP rows.
int two_stage_step(kimodo_ctx* c, int B, int T, int t, int t_prev, float w_cfg, int k_row, bool pack_next,
                   const Sampler& smp, const float* z_step, cudaStream_t st) {
  Workspace& w = c->ws;
  const int nseq = 2 * B, S = T + 1;
  const double eb = (double)c->elem();
  KD_TRY(run_net(c, 0, nseq, T, B, w.A_root, w.tmlp[0] + (long)k_row * D, w.txt[0], w.root_hat, st));
  KD_TRY(launch(c, CLS_MOTION, 0, (double)nseq * T * (ROOT_F * 4 + MOTION_F * (4 + eb)), st, "g2l_body_input", [&] {
    return g2l_body_input(w.root_hat, w.x, w.lengths, B, nseq, T, S, w.A_body, c->bf16(), BODY_IN_LD, st,
                          c->tk.packed ? w.tok0 : nullptr);
  }));
  KD_TRY(run_net(c, 1, nseq, T, B, w.A_body, w.tmlp[1] + (long)k_row * D, w.txt[1], w.body_hat, st));
  float c0, c1, c2;
  ddim_coeffs(c, smp.schedule, t, t_prev, smp.eta, &c0, &c1, &c2);
  const float* z = c2 != 0.f ? z_step : nullptr;
  return launch(c, CLS_MOTION, 0, (double)B * T * MOTION_F * 4 * (z ? 5 : 4), st, "cfg_ddim", [&] {
    return cfg_ddim(w.root_hat, w.body_hat, w.x, w.lengths, B, T, w_cfg, c0, c1, z, c2,
                    pack_next ? w.A_root : nullptr, c->bf16(), ROOT_IN_LD, S, st, c->tk.packed ? w.tok0 : nullptr);
  });
}

int pack_root_input(kimodo_ctx* c, int B, int nseq, int T, cudaStream_t st) {
  Workspace& w = c->ws;
  return launch(c, CLS_MOTION, 0, (double)nseq * T * ROOT_F * 8, st, "pack_frames", [&] {
    return pack_frames(w.x, B, MOTION_F, 0, ROOT_F, w.A_root, c->bf16(), ROOT_IN_LD, 0, nseq, T, T + 1, st,
                       c->tk.packed ? w.tok0 : nullptr, w.lengths, B);
  });
}

bool is_device_memory(const void* p);

// Chooses the token layout of a call (lengths already validated when on the host) and,
// for the packed layout, enqueues the token map built from the staged lengths.
Tokens plan_tokens(const int* lengths, int batch, int nseq, int frames) {
  Tokens tk;
  tk.M = nseq * (frames + 1);
  if (lengths != nullptr && !is_device_memory(lengths)) {
    long m = 0;
    for (int s = 0; s < nseq; ++s) m += 1 + lengths[s % batch];
    if (m < tk.M) {
      tk.M = (int)m;
      tk.packed = true;
    }
  }
  return tk;
}

int enqueue_token_map(kimodo_ctx* c, int batch, int nseq, cudaStream_t st) {
  if (!c->tk.packed) return KIMODO_OK;
  Workspace& w = c->ws;
  return launch(c, CLS_SETUP, 0, (double)c->tk.M * 4, st, "build_token_map",
                [&] { return build_token_map(w.lengths, batch, nseq, w.tok0, w.row_seq, st); });
}

// ------------------------------------------------------------------ argument checks

bool is_device_memory(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

int check_ctx(kimodo_ctx* c) {
  if (!c) return set_error(KIMODO_EINVAL, "ctx is NULL");
  KD_CUDA(cudaSetDevice(c->device));
  return KIMODO_OK;
}

int check_shape(int batch, int frames) {
  if (batch < 1) return set_error(KIMODO_EINVAL, "batch must be >= 1 (got %d)", batch);
  if (frames < 1 || frames > MAX_FRAMES)
    return set_error(KIMODO_EINVAL, "frames must be in [1, %d] (got %d)", MAX_FRAMES, frames);
  return KIMODO_OK;
}

// Host lengths are validated here; device lengths are used as given (kernels
// treat them as clamped to [0, frames]).
int stage_lengths(kimodo_ctx* c, const int* lengths, int batch, int frames, cudaStream_t st) {
  if (!lengths) return set_error(KIMODO_EINVAL, "lengths is NULL");
  if (!is_device_memory(lengths)) {
    for (int b = 0; b < batch; ++b)
      if (lengths[b] < 1 || lengths[b] > frames)
        return set_error(KIMODO_EINVAL, "lengths[%d] = %d outside [1, %d]", b, lengths[b], frames);
  }
  KD_CUDA(cudaMemcpyAsync(c->ws.lengths, lengths, (size_t)batch * 4, cudaMemcpyDefault, st));
  return KIMODO_OK;
}

const char* where_name(int where) {
  switch (where) {
    case WHERE_GEMM_PRODUCER: return "GEMM TMA producer";
    case WHERE_GEMM_MMA: return "GEMM MMA issuer";
    case WHERE_GEMM_EPILOGUE: return "GEMM epilogue";
    case WHERE_GEMM_DRAIN: return "GEMM MMA drain";
    case WHERE_ATTENTION: return "attention";
    case WHERE_WAIT_SELFTEST: return "wait self-test";
    default: return "unknown stage";
  }
}

// One CTA, one thread: a bounded wait on an mbarrier that nothing arrives on, with the
// same helper and the same error record as the GEMM and attention kernels.
__global__ void wait_selftest_kernel(DevError* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = ptx::smem_u32(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbar_init();
  volatile int abort = 0;
  if (!ptx::mbar_wait_bounded(b, 0, &abort, limit_ns) && atomicCAS(&err->code, 0, KIMODO_ETIMEOUT) == 0) {
    err->where = WHERE_WAIT_SELFTEST;
    err->block = blockIdx.x;
  }
}

int finish_outputs(kimodo_ctx* c, const void* out, cudaStream_t st) {
  if (!is_device_memory(out)) {
    KD_CUDA(cudaStreamSynchronize(st));
    DevError h;
    KD_CUDA(cudaMemcpy(&h, c->derr, sizeof(h), cudaMemcpyDeviceToHost));
    if (h.code != 0) {
      cudaMemset(c->derr, 0, sizeof(DevError));
      return set_error(h.code, "device wait timed out in %s (block %d)", where_name(h.where), h.block);
    }
  }
  return KIMODO_OK;
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* kimodo_last_error(void) { return g_last_error.c_str(); }

int kimodo_load_weights(kimodo_ctx** out_ctx, const float* host_blob, size_t n_floats, int precision, int device) {
  g_last_error.clear();
  if (!out_ctx) return set_error(KIMODO_EINVAL, "ctx out-pointer is NULL");
  *out_ctx = nullptr;
  if (!host_blob) return set_error(KIMODO_EINVAL, "weight blob is NULL");
  if (n_floats != (size_t)KIMODO_N_PARAMS)
    return set_error(KIMODO_EINVAL, "weight blob has %zu floats, expected %u", n_floats, KIMODO_N_PARAMS);
  if (precision != KIMODO_FP32 && precision != KIMODO_BF16)
    return set_error(KIMODO_EINVAL, "precision must be KIMODO_FP32 or KIMODO_BF16 (got %d)", precision);
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return set_error(KIMODO_EUNSUPPORTED, "no CUDA device available");
  }
  if (device < 0 || device >= ndev) return set_error(KIMODO_EINVAL, "device %d out of range [0, %d)", device, ndev);
  KD_CUDA(cudaSetDevice(device));
  cudaDeviceProp prop;
  KD_CUDA(cudaGetDeviceProperties(&prop, device));
  if (prop.major != 10)
    return set_error(KIMODO_EUNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", device,
                     prop.major, prop.minor);
  if (precision == KIMODO_BF16 && !gemm_tc_available())
    return set_error(KIMODO_EUNSUPPORTED, "cuTensorMapEncodeTiled is unavailable in this driver");

  if (gemm_tc_prepare() != cudaSuccess || gemm_tc2_prepare() != cudaSuccess || attention_tc_prepare() != cudaSuccess) {
    cudaGetLastError();
    return set_error(KIMODO_EUNSUPPORTED, "kernel attributes could not be set on device %d", device);
  }
  kimodo_ctx* c = new kimodo_ctx();
  c->device = device;
  c->precision = precision;
  c->num_sms = prop.multiProcessorCount;
  auto fail = [&](int code) {
    kimodo_free(c);
    return code;
  };
  cudaStream_t st;
  if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess)
    return fail(set_error(KIMODO_ECUDA, "stream creation failed"));
  c->cap_stream = st;

  // schedule and sinusoid table (double on the host)
  {
    double prod = 1.0;
    for (int i = 0; i < N_TRAIN; ++i) {
      const double beta = 1e-4 + (0.02 - 1e-4) * (double)i / (double)(N_TRAIN - 1);
      prod *= 1.0 - beta;
      c->alphabar[KIMODO_SCHEDULE_LINEAR][i] = prod;
    }
    // cosine (Nichol & Dhariwal 2021, eq. 17), s = 0.008, beta clipped at 0.999
    auto fcos = [](double u) {
      const double v = cos((u + 0.008) / 1.008 * M_PI / 2.0);
      return v * v;
    };
    prod = 1.0;
    for (int i = 0; i < N_TRAIN; ++i) {
      const double beta = fmin(1.0 - fcos((i + 1.0) / N_TRAIN) / fcos((double)i / N_TRAIN), 0.999);
      prod *= 1.0 - beta;
      c->alphabar[KIMODO_SCHEDULE_COSINE][i] = prod;
    }
    std::vector<float> pe((size_t)N_TRAIN * D);
    for (int p = 0; p < N_TRAIN; ++p)
      for (int i = 0; i < D / 2; ++i) {
        const double wv = pow(10000.0, -2.0 * i / (double)D);
        pe[(size_t)p * D + 2 * i] = (float)sin(p * wv);
        pe[(size_t)p * D + 2 * i + 1] = (float)cos(p * wv);
      }
    if (cudaMalloc(&c->pe, pe.size() * 4) != cudaSuccess) return fail(set_error(KIMODO_ENOMEM, "pe table"));
    if (cudaMemcpy(c->pe, pe.data(), pe.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(set_error(KIMODO_ECUDA, "pe upload"));
    if (cudaMalloc(&c->derr, sizeof(DevError)) != cudaSuccess) return fail(set_error(KIMODO_ENOMEM, "error word"));
    cudaMemset(c->derr, 0, sizeof(DevError));
  }

  // weights: plan the arena, stage the fp32 blob on the device, convert
  WeightWalker plan{c, nullptr, 0, nullptr, 0, st};
  plan.all();
  if (plan.src_off != (size_t)KIMODO_N_PARAMS) return fail(set_error(KIMODO_EINVAL, "internal layout mismatch"));
  if (cudaMalloc(&c->warena, plan.arena_off) != cudaSuccess)
    return fail(set_error(KIMODO_ENOMEM, "weight arena of %zu bytes", plan.arena_off));
  const float* dblob = host_blob;
  float* tmp = nullptr;
  if (!is_device_memory(host_blob)) {
    if (cudaMalloc(&tmp, n_floats * 4) != cudaSuccess) return fail(set_error(KIMODO_ENOMEM, "weight staging"));
    if (cudaMemcpy(tmp, host_blob, n_floats * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(tmp);
      return fail(set_error(KIMODO_ECUDA, "weight upload"));
    }
    dblob = tmp;
  }
  WeightWalker ww{c, dblob, 0, static_cast<char*>(c->warena), 0, st};
  ww.all();
  cudaError_t se = cudaStreamSynchronize(st);
  if (tmp) cudaFree(tmp);
  if (ww.err || se != cudaSuccess) return fail(set_error(KIMODO_ECUDA, "weight conversion failed"));
  *out_ctx = c;
  return KIMODO_OK;
}

void kimodo_free(kimodo_ctx* c) {
  if (!c) return;
  cudaSetDevice(c->device);
  free_graphs(c);
  for (auto e : c->ev_pool) cudaEventDestroy(e);
  if (c->ws.arena) cudaFree(c->ws.arena);
  for (int g = 0; g < SAMPLE_GROUPS; ++g) {
    if (c->gws[g].arena) cudaFree(c->gws[g].arena);
    if (c->gst[g]) cudaStreamDestroy(c->gst[g]);
  }
  for (int i = 0; i <= SAMPLE_GROUPS; ++i)
    if (c->gev[i]) cudaEventDestroy(c->gev[i]);
  if (c->zbuf) cudaFree(c->zbuf);
  if (c->warena) cudaFree(c->warena);
  if (c->pe) cudaFree(c->pe);
  if (c->derr) cudaFree(c->derr);
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  delete c;
}

int kimodo_denoiser_forward(kimodo_ctx* c, int net, const float* x, const float* emb, int t, const int* lengths,
                            int batch, int frames, float* out, void* stream) {
  g_last_error.clear();
  KD_TRY(check_ctx(c));
  if (net != KIMODO_NET_ROOT && net != KIMODO_NET_BODY) return set_error(KIMODO_EINVAL, "net must be 0 or 1");
  if (!x || !emb || !out) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  if (t < 0 || t >= N_TRAIN) return set_error(KIMODO_EINVAL, "t must be in [0, 999] (got %d)", t);
  KD_TRY(check_shape(batch, frames));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KD_TRY(ensure_workspace(c, batch, frames, 1));
  const long long l0 = c->launches;
  Workspace& w = c->ws;
  NetW& n = c->net[net];
  KD_TRY(stage_lengths(c, lengths, batch, frames, st));
  c->tk = plan_tokens(lengths, batch, batch, frames);
  KD_TRY(enqueue_token_map(c, batch, batch, st));
  KD_CUDA(cudaMemcpyAsync(w.x, x, (size_t)batch * frames * n.din * 4, cudaMemcpyDefault, st));
  KD_CUDA(cudaMemcpyAsync(w.st_text, emb, (size_t)batch * DTXT * 4, cudaMemcpyDefault, st));
  KD_TRY(launch(c, CLS_SETUP, 0, (double)batch * DTXT * 6, st, "pack_embeddings", [&] {
    return pack_embeddings(w.st_text, batch, nullptr, 1, 0, w.emb, c->bf16(), st);
  }));
  KD_TRY(timestep_rows(c, t, 0, 1, st));
  KD_TRY(condition_setup(c, net, batch, 1, st));
  void* A = net == 0 ? w.A_root : w.A_body;
  const int lda = net == 0 ? ROOT_IN_LD : BODY_IN_LD;
  KD_TRY(launch(c, CLS_MOTION, 0, (double)batch * frames * n.din * 8, st, "pack_frames", [&] {
    return pack_frames(w.x, batch, n.din, 0, n.din, A, c->bf16(), lda, 0, batch, frames, frames + 1, st,
                       c->tk.packed ? w.tok0 : nullptr, w.lengths, batch);
  }));
  float* hat = net == 0 ? w.root_hat : w.body_hat;
  // the packed layout has no rows for padded frames: their outputs are the zeros set here
  if (c->tk.packed) KD_CUDA(cudaMemsetAsync(hat, 0, (size_t)batch * frames * n.dout * 4, st));
  KD_TRY(run_net(c, net, batch, frames, batch, A, w.tmlp[net], w.txt[net], hat, st));
  KD_CUDA(cudaMemcpyAsync(out, hat, (size_t)batch * frames * n.dout * 4, cudaMemcpyDefault, st));
  c->last_launches = c->launches - l0;
  return finish_outputs(c, out, st);
}

// Validates the sampler options; n_z = floats of step noise the call reads when eta > 0.
static int check_sampler(kimodo_ctx* c, const kimodo_sampler* o, int batch, size_t n_z, Sampler* out,
                         cudaStream_t st) {
  *out = Sampler();
  if (!o) return KIMODO_OK;
  if (o->text_batch != 0) {
    if (o->text_batch < 1 || o->text_batch > batch || batch % o->text_batch)
      return set_error(KIMODO_EINVAL, "text_batch must divide batch (got %d for batch %d)", o->text_batch, batch);
    out->takes = batch / o->text_batch;
  }
  if (o->schedule != KIMODO_SCHEDULE_LINEAR && o->schedule != KIMODO_SCHEDULE_COSINE)
    return set_error(KIMODO_EINVAL, "unknown schedule %d", o->schedule);
  if (!isfinite(o->eta) || o->eta < 0.f || o->eta > 1.f)
    return set_error(KIMODO_EINVAL, "eta must be in [0, 1]");
  out->schedule = o->schedule;
  out->eta = o->eta;
  if (o->eta == 0.f) return KIMODO_OK;
  if (!o->step_noise) return set_error(KIMODO_EINVAL, "eta > 0 needs step_noise");
  if (is_device_memory(o->step_noise)) {
    out->z = o->step_noise;
    return KIMODO_OK;
  }
  if (c->zcap < n_z) {   // host draws: staged into a context buffer that only grows
    if (c->zbuf) {
      KD_CUDA(cudaStreamSynchronize(st));
      cudaFree(c->zbuf);
      c->zbuf = nullptr;
      c->zcap = 0;
    }
    if (cudaMalloc(&c->zbuf, n_z * 4) != cudaSuccess) return set_error(KIMODO_ENOMEM, "step noise staging");
    c->zcap = n_z;
  }
  KD_CUDA(cudaMemcpyAsync(c->zbuf, o->step_noise, n_z * 4, cudaMemcpyHostToDevice, st));
  out->z = c->zbuf;
  return KIMODO_OK;
}

int kimodo_ddim_step(kimodo_ctx* c, const float* x_t, const float* text_emb, const float* null_emb, int null_batch,
                     const int* lengths, int batch, int frames, int t, int t_prev, float cfg_scale, float* x_prev,
                     void* stream) {
  return kimodo_ddim_step_ex(c, x_t, text_emb, null_emb, null_batch, lengths, batch, frames, t, t_prev, cfg_scale,
                             nullptr, x_prev, stream);
}

int kimodo_ddim_step_ex(kimodo_ctx* c, const float* x_t, const float* text_emb, const float* null_emb,
                        int null_batch, const int* lengths, int batch, int frames, int t, int t_prev,
                        float cfg_scale, const kimodo_sampler* options, float* x_prev, void* stream) {
  g_last_error.clear();
  KD_TRY(check_ctx(c));
  if (!x_t || !text_emb || !null_emb || !x_prev) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  KD_TRY(check_shape(batch, frames));
  if (t < 0 || t >= N_TRAIN) return set_error(KIMODO_EINVAL, "t must be in [0, 999] (got %d)", t);
  if (t_prev < -1 || t_prev >= t) return set_error(KIMODO_EINVAL, "t_prev must be in [-1, t) (got %d)", t_prev);
  if (!isfinite(cfg_scale)) return set_error(KIMODO_EINVAL, "cfg_scale must be finite");
  if (null_batch != 1 && null_batch != batch)
    return set_error(KIMODO_EINVAL, "null_batch must be 1 or batch (got %d)", null_batch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Sampler smp;
  KD_TRY(check_sampler(c, options, batch, (size_t)batch * frames * MOTION_F, &smp, st));
  KD_TRY(ensure_workspace(c, 2 * batch, frames, 1));
  const long long l0 = c->launches;
  Workspace& w = c->ws;
  KD_TRY(stage_lengths(c, lengths, batch, frames, st));
  c->tk = plan_tokens(lengths, batch, 2 * batch, frames);
  KD_TRY(enqueue_token_map(c, batch, 2 * batch, st));
  KD_CUDA(cudaMemcpyAsync(w.x, x_t, (size_t)batch * frames * MOTION_F * 4, cudaMemcpyDefault, st));
  KD_CUDA(cudaMemcpyAsync(w.st_text, text_emb, (size_t)(batch / smp.takes) * DTXT * 4, cudaMemcpyDefault, st));
  KD_CUDA(cudaMemcpyAsync(w.st_null, null_emb, (size_t)null_batch * DTXT * 4, cudaMemcpyDefault, st));
  KD_TRY(launch(c, CLS_SETUP, 0, (double)2 * batch * DTXT * 6, st, "pack_embeddings", [&] {
    return pack_embeddings(w.st_text, batch, w.st_null, null_batch, batch, w.emb, c->bf16(), st, smp.takes);
  }));
  KD_TRY(timestep_rows(c, t, 0, 1, st));
  KD_TRY(condition_setup(c, 0, 2 * batch, 1, st));
  KD_TRY(condition_setup(c, 1, 2 * batch, 1, st));
  KD_TRY(pack_root_input(c, batch, 2 * batch, frames, st));
  KD_TRY(two_stage_step(c, batch, frames, t, t_prev, cfg_scale, 0, false, smp, smp.z, st));
  KD_CUDA(cudaMemcpyAsync(x_prev, w.x, (size_t)batch * frames * MOTION_F * 4, cudaMemcpyDefault, st));
  c->last_launches = c->launches - l0;
  return finish_outputs(c, x_prev, st);
}

// The sampling loop of `batch` prompts on the current workspace: set-up, then `steps`
// two-stage steps.  Step draws z (eta > 0) are read at prompt offset b0 of a call of
// batch_all prompts ([steps, batch_all, frames, 279]).
static int enqueue_loop(kimodo_ctx* c, int batch, int frames, int steps, float cfg, int null_batch,
                        const Sampler& smp, int b0, int batch_all, cudaStream_t st) {
  Workspace& w = c->ws;
  KD_TRY(enqueue_token_map(c, batch, 2 * batch, st));
  KD_TRY(launch(c, CLS_SETUP, 0, (double)2 * batch * DTXT * 6, st, "pack_embeddings", [&] {
    return pack_embeddings(w.st_text, batch, w.st_null, null_batch, batch, w.emb, c->bf16(), st, smp.takes);
  }));
  KD_TRY(timestep_rows(c, -1, steps, steps, st));
  KD_TRY(condition_setup(c, 0, 2 * batch, steps, st));
  KD_TRY(condition_setup(c, 1, 2 * batch, steps, st));
  KD_TRY(pack_root_input(c, batch, 2 * batch, frames, st));
  const size_t zstep = (size_t)batch_all * frames * MOTION_F;
  for (int k = 0; k < steps; ++k) {
    const float* z = smp.z ? smp.z + k * zstep + (size_t)b0 * frames * MOTION_F : nullptr;
    KD_TRY(two_stage_step(c, batch, frames, trailing_t(k, steps), trailing_t(k + 1, steps), cfg, k, k + 1 < steps,
                          smp, z, st));
  }
  return KIMODO_OK;
}

// Prompt groups for a call: SAMPLE_GROUPS when the prompts split evenly (takes of one
// prompt stay together) and every group keeps GROUP_MIN_ROWS token rows, else 1.
static int sample_groups(const kimodo_ctx* c, int batch, const Sampler& smp) {
  if (SAMPLE_GROUPS < 2 || c->profiling || batch % SAMPLE_GROUPS) return 1;
  const int bg = batch / SAMPLE_GROUPS;
  if (bg % smp.takes) return 1;
  return 2 * bg * (c->tk.M / (2 * batch)) >= GROUP_MIN_ROWS ? SAMPLE_GROUPS : 1;
}

static int ensure_group_resources(kimodo_ctx* c, int groups, int batch, int frames, int steps) {
  for (int g = 0; g < groups; ++g) {
    bool grown = false;
    KD_TRY(alloc_workspace(c, c->gws[g], 2 * (batch / groups), frames, steps, &grown));
    if (grown) free_graphs(c);
    if (!c->gst[g] && cudaStreamCreateWithFlags(&c->gst[g], cudaStreamNonBlocking) != cudaSuccess)
      return set_error(KIMODO_ECUDA, "stream creation failed");
  }
  for (int i = 0; i <= groups; ++i)
    if (!c->gev[i] && cudaEventCreateWithFlags(&c->gev[i], cudaEventDisableTiming) != cudaSuccess)
      return set_error(KIMODO_ECUDA, "event creation failed");
  return KIMODO_OK;
}

// The whole sampling call.  With prompt groups, each group's loop is enqueued on its own
// stream (forked from st and joined back, so a capture on st records them as parallel
// graph branches) on its own workspace; the state x, lengths and embedding staging are
// the call's, viewed at the group's prompt offset.
static int enqueue_sample(kimodo_ctx* c, int batch, int frames, int steps, float cfg, int null_batch,
                          const Sampler& smp, const int* lengths, cudaStream_t st) {
  const int groups = sample_groups(c, batch, smp);
  if (groups == 1) return enqueue_loop(c, batch, frames, steps, cfg, null_batch, smp, 0, batch, st);
  const Workspace main_ws = c->ws;
  const Tokens main_tk = c->tk;
  const int bg = batch / groups;
  KD_CUDA(cudaEventRecord(c->gev[0], st));
  int r = KIMODO_OK;
  for (int g = 0; g < groups && r == KIMODO_OK; ++g) {
    const int b0 = g * bg;
    Workspace w = c->gws[g];
    w.x = main_ws.x + (size_t)b0 * frames * MOTION_F;
    w.lengths = main_ws.lengths + b0;
    w.st_text = main_ws.st_text + (size_t)(b0 / smp.takes) * DTXT;
    w.st_null = main_ws.st_null + (null_batch == 1 ? 0 : (size_t)b0 * DTXT);
    c->ws = w;
    c->tk = plan_tokens(lengths + b0, bg, 2 * bg, frames);
    if (cudaStreamWaitEvent(c->gst[g], c->gev[0], 0) != cudaSuccess) {
      r = set_error(KIMODO_ECUDA, "stream fork failed");
      break;
    }
    r = enqueue_loop(c, bg, frames, steps, cfg, null_batch == 1 ? 1 : bg, smp, b0, batch, c->gst[g]);
    if (r == KIMODO_OK && (cudaEventRecord(c->gev[1 + g], c->gst[g]) != cudaSuccess ||
                           cudaStreamWaitEvent(st, c->gev[1 + g], 0) != cudaSuccess))
      r = set_error(KIMODO_ECUDA, "stream join failed");
  }
  c->ws = main_ws;
  c->tk = main_tk;
  return r;
}

int kimodo_ddim_sample(kimodo_ctx* c, const float* text_emb, const float* null_emb, int null_batch,
                       const float* noise, const int* lengths, int batch, int frames, int steps, float cfg_scale,
                       float* out, void* stream) {
  return kimodo_ddim_sample_ex(c, text_emb, null_emb, null_batch, noise, lengths, batch, frames, steps, cfg_scale,
                               nullptr, out, stream);
}

int kimodo_ddim_sample_ex(kimodo_ctx* c, const float* text_emb, const float* null_emb, int null_batch,
                          const float* noise, const int* lengths, int batch, int frames, int steps, float cfg_scale,
                          const kimodo_sampler* options, float* out, void* stream) {
  g_last_error.clear();
  KD_TRY(check_ctx(c));
  if (!text_emb || !null_emb || !noise || !out) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  KD_TRY(check_shape(batch, frames));
  if (steps < 1 || steps > N_TRAIN) return set_error(KIMODO_EINVAL, "steps must be in [1, %d] (got %d)", N_TRAIN, steps);
  if (!isfinite(cfg_scale)) return set_error(KIMODO_EINVAL, "cfg_scale must be finite");
  if (null_batch != 1 && null_batch != batch)
    return set_error(KIMODO_EINVAL, "null_batch must be 1 or batch (got %d)", null_batch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Sampler smp;
  KD_TRY(check_sampler(c, options, batch, (size_t)steps * batch * frames * MOTION_F, &smp, st));
  KD_TRY(ensure_workspace(c, 2 * batch, frames, steps));
  Workspace& w = c->ws;
  KD_TRY(stage_lengths(c, lengths, batch, frames, st));
  c->tk = plan_tokens(lengths, batch, 2 * batch, frames);
  // the prompt groups' workspaces and streams exist before any capture begins
  const int groups = sample_groups(c, batch, smp);
  if (groups > 1) KD_TRY(ensure_group_resources(c, groups, batch, frames, steps));
  KD_CUDA(cudaMemcpyAsync(w.x, noise, (size_t)batch * frames * MOTION_F * 4, cudaMemcpyDefault, st));
  KD_CUDA(cudaMemcpyAsync(w.st_text, text_emb, (size_t)(batch / smp.takes) * DTXT * 4, cudaMemcpyDefault, st));
  KD_CUDA(cudaMemcpyAsync(w.st_null, null_emb, (size_t)null_batch * DTXT * 4, cudaMemcpyDefault, st));
  const long long l0 = c->launches;
  if (c->profiling) {
    // The profiled generation runs as a graph too, with a timing event node on
    // each side of every kernel node, so per-kernel times carry no host gaps.
    // The graph is not cached: its event nodes belong to this profile.
    KD_CUDA(cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal));
    c->prof_flags = cudaEventRecordExternal;
    int s = enqueue_sample(c, batch, frames, steps, cfg_scale, null_batch, smp, lengths, c->cap_stream);
    c->prof_flags = cudaEventRecordDefault;
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(c->cap_stream, &g);
    if (s != KIMODO_OK) {
      if (g) cudaGraphDestroy(g);
      return s;
    }
    if (e != cudaSuccess) return set_error(KIMODO_ECUDA, "graph capture failed: %s", cudaGetErrorString(e));
    cudaGraphExec_t ge;
    e = cudaGraphInstantiate(&ge, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return set_error(KIMODO_ECUDA, "graph instantiate failed: %s", cudaGetErrorString(e));
    e = cudaGraphLaunch(ge, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    cudaGraphExecDestroy(ge);
    if (e != cudaSuccess) return set_error(KIMODO_ECUDA, "profiled graph failed: %s", cudaGetErrorString(e));
    c->last_launches = c->launches - l0;
  } else {
    uint32_t cfg_bits, eta_bits;
    memcpy(&cfg_bits, &cfg_scale, 4);
    memcpy(&eta_bits, &smp.eta, 4);
    const auto key = std::make_tuple(batch, frames, steps, (null_batch == 1 ? 1 : 0) | (smp.takes << 1), cfg_bits,
                                     smp.schedule, eta_bits, smp.z, c->tk.packed ? c->tk.M : -1);
    auto it = c->graphs.find(key);
    if (it == c->graphs.end()) {
      KD_CUDA(cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal));
      const long long lc = c->launches;
      int s = enqueue_sample(c, batch, frames, steps, cfg_scale, null_batch, smp, lengths, c->cap_stream);
      cudaGraph_t g = nullptr;
      cudaError_t e = cudaStreamEndCapture(c->cap_stream, &g);
      if (s != KIMODO_OK) {
        if (g) cudaGraphDestroy(g);
        return s;
      }
      if (e != cudaSuccess) return set_error(KIMODO_ECUDA, "graph capture failed: %s", cudaGetErrorString(e));
      cudaGraphExec_t ge;
      e = cudaGraphInstantiate(&ge, g, 0);
      cudaGraphDestroy(g);
      if (e != cudaSuccess) return set_error(KIMODO_ECUDA, "graph instantiate failed: %s", cudaGetErrorString(e));
      it = c->graphs.emplace(key, std::make_pair(ge, c->launches - lc)).first;
    }
    KD_CUDA(cudaGraphLaunch(it->second.first, st));
    c->last_launches = it->second.second;
  }
  KD_CUDA(cudaMemcpyAsync(out, w.x, (size_t)batch * frames * MOTION_F * 4, cudaMemcpyDefault, st));
  return finish_outputs(c, out, st);
}

int kimodo_sync_status(kimodo_ctx* c, void* stream) {
  g_last_error.clear();
  KD_TRY(check_ctx(c));
  KD_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  DevError h;
  KD_CUDA(cudaMemcpy(&h, c->derr, sizeof(h), cudaMemcpyDeviceToHost));
  if (h.code != 0) {
    KD_CUDA(cudaMemset(c->derr, 0, sizeof(DevError)));
    return set_error(h.code, "device wait timed out in %s (block %d)", where_name(h.where), h.block);
  }
  return KIMODO_OK;
}

int kimodo_wait_selftest(kimodo_ctx* c, int limit_us, void* stream) {
  g_last_error.clear();
  KD_TRY(check_ctx(c));
  if (limit_us < 1 || limit_us > 2000000) return set_error(KIMODO_EINVAL, "limit_us must be in [1, 2000000]");
  wait_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(c->derr, 1000ull * (unsigned)limit_us);
  KD_CUDA(cudaGetLastError());
  return KIMODO_OK;
}

int kimodo_profile_enable(kimodo_ctx* c, int enable) {
  g_last_error.clear();
  if (!c) return set_error(KIMODO_EINVAL, "ctx is NULL");
  c->profiling = enable != 0;
  c->prof.clear();
  c->ev_used = 0;
  return KIMODO_OK;
}

int kimodo_profile_read(kimodo_ctx* c, int n_classes, double* ms, long long* launches, double* flops,
                        double* bytes) {
  g_last_error.clear();
  KD_TRY(check_ctx(c));
  if (n_classes < 1 || n_classes > NUM_CLS) return set_error(KIMODO_EINVAL, "n_classes must be in [1, 8]");
  for (int i = 0; i < n_classes; ++i) {
    if (ms) ms[i] = 0;
    if (launches) launches[i] = 0;
    if (flops) flops[i] = 0;
    if (bytes) bytes[i] = 0;
  }
  KD_CUDA(cudaDeviceSynchronize());
  for (auto& r : c->prof) {
    if (r.cls >= n_classes) continue;
    float t = 0;
    KD_CUDA(cudaEventElapsedTime(&t, r.a, r.b));
    if (ms) ms[r.cls] += t;
    if (launches) launches[r.cls] += 1;
    if (flops) flops[r.cls] += r.flops;
    if (bytes) bytes[r.cls] += r.bytes;
  }
  c->prof.clear();
  c->ev_used = 0;
  return KIMODO_OK;
}

long long kimodo_last_launch_count(kimodo_ctx* c) { return c ? c->last_launches : 0; }

}  // extern "C"

// ====================================================================== kernel-level entry points

namespace {

DevError* kernel_error_word() {
  static DevError* p[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!p[dev] && cudaMalloc(&p[dev], sizeof(DevError)) == cudaSuccess) cudaMemset(p[dev], 0, sizeof(DevError));
  return p[dev];
}

int prepared_device() {
  static bool done[64] = {};
  int dev = 0;
  KD_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return set_error(KIMODO_EINVAL, "device index");
  if (!done[dev]) {
    KD_CUDA(gemm_tc_prepare());
    KD_CUDA(gemm_tc2_prepare());
    KD_CUDA(attention_tc_prepare());
    done[dev] = true;
  }
  return KIMODO_OK;
}

int check_gemm_args(const void* A, int lda, const void* W, int ldw, const float* bias, const void* resid, void* out,
                    int ldo, int M, int N, int K, int epi) {
  if (!A || !W || !bias || !out) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  if (M < 1 || N < 1 || K < 1) return set_error(KIMODO_EINVAL, "M, N, K must be >= 1");
  if (lda < K || ldw < K || ldo < N) return set_error(KIMODO_EINVAL, "leading dimensions must cover K / N");
  if (epi < 0 || epi > 3) return set_error(KIMODO_EINVAL, "unknown epilogue %d", epi);
  if (epi == 3 && !resid) return set_error(KIMODO_EINVAL, "residual epilogue needs resid");
  return KIMODO_OK;
}

}  // namespace

extern "C" {

int kimodo_gemm_bf16(const void* A, int lda, const void* W, int ldw, const float* bias, const void* resid, int ldr,
                     void* out, int ldo, int M, int N, int K, int epilogue, int out_f32, int tile_n, void* stream) {
  g_last_error.clear();
  KD_TRY(check_gemm_args(A, lda, W, ldw, bias, resid, out, ldo, M, N, K, epilogue));
  if (lda % 8 || ldw % 8 || (reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(W) & 15))
    return set_error(KIMODO_EINVAL, "bf16 operands need 16-byte aligned rows (lda, ldw multiples of 8)");
  if (ldo % 4 || (reinterpret_cast<uintptr_t>(out) & 15) || (epilogue == 3 && (ldr % 4 ||
      (reinterpret_cast<uintptr_t>(resid) & 15))) || (reinterpret_cast<uintptr_t>(bias) & 15))
    return set_error(KIMODO_EINVAL, "out, resid and bias need 16-byte alignment and ldo, ldr multiples of 4");
  if (epilogue == 3 && !out_f32) return set_error(KIMODO_EINVAL, "residual epilogue writes fp32");
  if ((epilogue == 1 || epilogue == 2) && out_f32) return set_error(KIMODO_EINVAL, "GELU/SiLU epilogues write bf16");
  if (tile_n != 0 && tile_n != 32 && tile_n != 64 && tile_n != 128 && tile_n != 256)
    return set_error(KIMODO_EINVAL, "tile_n must be 0, 32, 64, 128 or 256");
  if (tile_n == 256 && (epilogue == KIMODO_EPI_BIAS_SILU || (out_f32 && epilogue == KIMODO_EPI_BIAS)))
    return set_error(KIMODO_EINVAL, "tile_n 256 is not built for this epilogue");
  if ((tile_n == 32 || tile_n == 64) && (epilogue == KIMODO_EPI_BIAS_SILU || (out_f32 && epilogue == KIMODO_EPI_BIAS)))
    return set_error(KIMODO_EINVAL, "tile_n 32 and 64 are not built for this epilogue");
  KD_TRY(prepared_device());
  int dev = 0, sms = 148;
  KD_CUDA(cudaGetDevice(&dev));
  KD_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  GemmArgs g;
  g.A = A; g.B = W; g.M = M; g.N = N; g.K = K; g.lda = lda; g.ldb = ldw;
  EpiParams ep;
  ep.bias = bias; ep.out = out; ep.ldo = ldo; ep.resid = resid; ep.ldr = ldr; ep.N = N; ep.M = M;
  const int bn = tile_n ? tile_n : 128;
  KD_CUDA(gemm_tc(g, bn, epilogue, out_f32 != 0, ep, kernel_error_word(), static_cast<cudaStream_t>(stream), sms));
  return KIMODO_OK;
}

int kimodo_gemm_bf16_pair(const void* A, int lda, const void* W, int ldw, const float* bias, const void* resid,
                          int ldr, void* out, int ldo, int M, int N, int K, int epilogue, int out_f32, int tile_n,
                          void* stream) {
  g_last_error.clear();
  KD_TRY(check_gemm_args(A, lda, W, ldw, bias, resid, out, ldo, M, N, K, epilogue));
  if (lda % 8 || ldw % 8 || (reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(W) & 15))
    return set_error(KIMODO_EINVAL, "bf16 operands need 16-byte aligned rows (lda, ldw multiples of 8)");
  if (ldo % 4 || (reinterpret_cast<uintptr_t>(out) & 15) || (epilogue == 3 && (ldr % 4 ||
      (reinterpret_cast<uintptr_t>(resid) & 15))) || (reinterpret_cast<uintptr_t>(bias) & 15))
    return set_error(KIMODO_EINVAL, "out, resid and bias need 16-byte alignment and ldo, ldr multiples of 4");
  if (!gemm_tc2_supports(epilogue, out_f32 != 0))
    return set_error(KIMODO_EINVAL, "pair GEMM epilogues: bias or GELU with bf16 output, residual with fp32 output");
  if (N % 16 || ((long)ldo * (out_f32 ? 4 : 2)) % 16)
    return set_error(KIMODO_EINVAL, "pair GEMM needs N % 16 == 0 and 16-byte output rows");
  if (tile_n != 0 && tile_n != 144 && tile_n != 160 && tile_n != 208 && tile_n != 256)
    return set_error(KIMODO_EINVAL, "tile_n must be 0, 144, 160, 208 or 256");
  if (epilogue == KIMODO_EPI_BIAS_RESID && tile_n > 160)
    return set_error(KIMODO_EINVAL, "the residual epilogue is built for tile_n 144 and 160");
  KD_TRY(prepared_device());
  GemmArgs g;
  g.A = A; g.B = W; g.M = M; g.N = N; g.K = K; g.lda = lda; g.ldb = ldw;
  EpiParams ep;
  ep.bias = bias; ep.out = out; ep.ldo = ldo; ep.resid = resid; ep.ldr = ldr; ep.N = N; ep.M = M;
  const int bn = tile_n ? tile_n : gemm_tc2_pick_bn(M, N, epilogue);
  KD_CUDA(gemm_tc2(g, bn, epilogue, out_f32 != 0, ep, kernel_error_word(), static_cast<cudaStream_t>(stream)));
  return KIMODO_OK;
}

int kimodo_gemm_f32(const float* A, int lda, const float* W, int ldw, const float* bias, const float* resid, int ldr,
                    float* out, int ldo, int M, int N, int K, int epilogue, void* stream) {
  g_last_error.clear();
  KD_TRY(check_gemm_args(A, lda, W, ldw, bias, resid, out, ldo, M, N, K, epilogue));
  if (K % 16 || lda % 4 || ldw % 4) return set_error(KIMODO_EINVAL, "fp32 GEMM needs K % 16 == 0, lda/ldw % 4 == 0");
  GemmArgs g;
  g.A = A; g.B = W; g.M = M; g.N = N; g.K = K; g.lda = lda; g.ldb = ldw;
  EpiParams ep;
  ep.bias = bias; ep.out = out; ep.ldo = ldo; ep.resid = resid; ep.ldr = ldr; ep.N = N; ep.M = M;
  KD_CUDA(gemm_f32(g, epilogue, ep, static_cast<cudaStream_t>(stream)));
  return KIMODO_OK;
}

int kimodo_attention_bf16(const void* qkv, void* out, const int* lengths, int nseq, int S, void* stream) {
  g_last_error.clear();
  if (!qkv || !out || !lengths) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  if (nseq < 1 || S < 1 || S > MAX_FRAMES + 1) return set_error(KIMODO_EINVAL, "need nseq >= 1, 1 <= S <= 301");
  if (reinterpret_cast<uintptr_t>(qkv) & 15) return set_error(KIMODO_EINVAL, "qkv must be 16-byte aligned");
  KD_TRY(prepared_device());
  KD_CUDA(attention_tc(static_cast<const bf16*>(qkv), static_cast<bf16*>(out), nseq * S, lengths, nseq, nseq, S,
                       kernel_error_word(), static_cast<cudaStream_t>(stream)));
  return KIMODO_OK;
}

int kimodo_attention_f32(const float* qkv, float* out, const int* lengths, int nseq, int S, void* stream) {
  g_last_error.clear();
  if (!qkv || !out || !lengths) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  if (nseq < 1 || S < 1 || S > MAX_FRAMES + 1) return set_error(KIMODO_EINVAL, "need nseq >= 1, 1 <= S <= 301");
  KD_CUDA(attention_f32(qkv, out, lengths, nseq, nseq, S, static_cast<cudaStream_t>(stream)));
  return KIMODO_OK;
}

int kimodo_layernorm(const float* y, void* out, int out_bf16, const float* gamma, const float* beta, int M,
                     void* stream) {
  g_last_error.clear();
  if (!y || !out || !gamma || !beta) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  if (M < 1) return set_error(KIMODO_EINVAL, "M must be >= 1");
  KD_CUDA(layernorm(y, out, out_bf16 != 0, gamma, beta, M, static_cast<cudaStream_t>(stream)));
  return KIMODO_OK;
}

int kimodo_global_to_local_root(const float* root, const float* x, const int* lengths, int batch, int frames,
                                float* body_in, void* stream) {
  g_last_error.clear();
  if (!root || !x || !lengths || !body_in) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  KD_TRY(check_shape(batch, frames));
  // The kernel places frame i of sequence s at row s * S + 1 + i of its output matrix
  // (row s * S is the condition token).  With S = frames and the base one row before
  // body_in, that row is body_in's row s * frames + i; row 0 itself is never written.
  float* base = body_in - MOTION_F;
  KD_CUDA(g2l_body_input(root, x, lengths, batch, batch, frames, frames, base, false, MOTION_F,
                         static_cast<cudaStream_t>(stream)));
  return KIMODO_OK;
}

}  // extern "C"

// ====================================================================== allocation-free forward
//
// kimodo_denoiser_forward_noalloc runs the same kernels as kimodo_denoiser_forward,
// but its activation workspace is the file-scope device array below instead of the
// context's lazily cudaMalloc'ed workspace.  The array is sized for the largest
// call it accepts (NOALLOC_MAX_ROWS tokens, NOALLOC_MAX_BATCH sequences, fp32
// elements, which bounds the bf16 layout too).  Its device address is looked up
// once per device with cudaGetSymbolAddress, on the first call made on that device.

namespace {

constexpr int NOALLOC_MAX_ROWS = 512;    // batch * (frames + 1)
constexpr int NOALLOC_MAX_BATCH = 16;

// Lays out a Workspace for (rows, nseq, nseq*frames) with element size e starting
// at `base`; returns the bytes used.  With base == nullptr it only measures.
constexpr size_t noalloc_layout(char* base, size_t e, size_t rows, size_t nseq, size_t nframes, Workspace* w) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += (bytes + 255) & ~size_t(255);
    return p;
  };
  char* h = take(rows * D * e);
  char* qkv = take(rows * 3 * D * e);
  char* attn = take(rows * D * e);
  char* u = take(rows * F * e);
  char* y = take(rows * D * 4);
  char* ar = take(rows * ROOT_IN_LD * e);
  char* ab = take(rows * BODY_IN_LD * e);
  char* rh = take(nframes * ROOT_F * 4);
  char* bh = take(nframes * BODY_F * 4);
  char* x = take(nframes * MOTION_F * 4);
  char* emb = take(nseq * DTXT * e);
  char* txt0 = take(nseq * D * 4);
  char* txt1 = take(nseq * D * 4);
  char* tpe = take(D * e);
  char* thid = take(D * e);
  char* tm0 = take(D * 4);
  char* tm1 = take(D * 4);
  char* len = take(nseq * 4);
  char* stt = take(nseq * DTXT * 4);
  char* st0 = take(rows * 8);
  char* st1 = take(rows * 8);
  if (w) {
    w->h = h; w->qkv = qkv; w->attn = attn; w->u = u; w->y = reinterpret_cast<float*>(y);
    w->A_root = ar; w->A_body = ab;
    w->root_hat = reinterpret_cast<float*>(rh); w->body_hat = reinterpret_cast<float*>(bh);
    w->x = reinterpret_cast<float*>(x); w->emb = emb;
    w->txt[0] = reinterpret_cast<float*>(txt0); w->txt[1] = reinterpret_cast<float*>(txt1);
    w->tpe = tpe; w->thid = thid;
    w->tmlp[0] = reinterpret_cast<float*>(tm0); w->tmlp[1] = reinterpret_cast<float*>(tm1);
    w->lengths = reinterpret_cast<int*>(len); w->st_text = reinterpret_cast<float*>(stt); w->st_null = nullptr;
    w->stats[0] = reinterpret_cast<float*>(st0); w->stats[1] = reinterpret_cast<float*>(st1);
  }
  return off;
}

constexpr size_t NOALLOC_BYTES =
    noalloc_layout(nullptr, 4, NOALLOC_MAX_ROWS, NOALLOC_MAX_BATCH, NOALLOC_MAX_ROWS, nullptr);

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_BYTES];

namespace {

// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name stands for a host-side shadow, not the device memory, so the address is looked up
// once per device (set-up, with that device current) and cached; the lookup is serialised
// so that threads making their first call at the same time agree on it.
int noalloc_scratch(char** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  KD_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return set_error(KIMODO_EINVAL, "device index %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return set_error(KIMODO_ECUDA, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
    }
    addr[dev] = p;
  }
  *out = static_cast<char*>(addr[dev]);
  return KIMODO_OK;
}

// Restores the context's own workspace and profiling flag on every exit path.
struct WorkspaceSwap {
  kimodo_ctx* c;
  Workspace saved;
  bool prof;
  WorkspaceSwap(kimodo_ctx* ctx, const Workspace& w) : c(ctx), saved(ctx->ws), prof(ctx->profiling) {
    c->ws = w;
    c->profiling = false;
  }
  ~WorkspaceSwap() {
    c->ws = saved;
    c->profiling = prof;
  }
};

}  // namespace

extern "C" int kimodo_denoiser_forward_noalloc(kimodo_ctx* c, int net, const float* x, const float* emb, int t,
                                               const int* lengths, int batch, int frames, float* out,
                                               void* stream) {
  g_last_error.clear();
  KD_TRY(check_ctx(c));
  if (net != KIMODO_NET_ROOT && net != KIMODO_NET_BODY) return set_error(KIMODO_EINVAL, "net must be 0 or 1");
  if (!x || !emb || !out) return set_error(KIMODO_EINVAL, "NULL tensor argument");
  if (t < 0 || t >= N_TRAIN) return set_error(KIMODO_EINVAL, "t must be in [0, 999] (got %d)", t);
  KD_TRY(check_shape(batch, frames));
  if (batch > NOALLOC_MAX_BATCH || (long)batch * (frames + 1) > NOALLOC_MAX_ROWS)
    return set_error(KIMODO_EINVAL,
                     "kimodo_denoiser_forward_noalloc: batch %d x (frames %d + 1) exceeds its static scratch "
                     "(at most %d sequences and %d tokens); use kimodo_denoiser_forward",
                     batch, frames, NOALLOC_MAX_BATCH, NOALLOC_MAX_ROWS);
  char* base = nullptr;
  KD_TRY(noalloc_scratch(&base));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = batch * (frames + 1);
  Workspace w;
  const size_t used = noalloc_layout(base, c->elem(), rows, batch, (size_t)batch * frames, &w);
  if (used > NOALLOC_BYTES) return set_error(KIMODO_EINVAL, "internal: static scratch layout overflow");
  WorkspaceSwap swap(c, w);
  const long long l0 = c->launches;
  NetW& n = c->net[net];
  // the scratch keeps the previous call's contents: the zero-padded K columns of
  // the input matrices must read as 0, so clear both matrices
  KD_CUDA(cudaMemsetAsync(w.A_root, 0, (size_t)rows * ROOT_IN_LD * c->elem(), st));
  KD_CUDA(cudaMemsetAsync(w.A_body, 0, (size_t)rows * BODY_IN_LD * c->elem(), st));
  KD_TRY(stage_lengths(c, lengths, batch, frames, st));
  c->tk = Tokens{rows, false};   // the scratch holds the padded layout only
  KD_CUDA(cudaMemcpyAsync(w.x, x, (size_t)batch * frames * n.din * 4, cudaMemcpyDefault, st));
  KD_CUDA(cudaMemcpyAsync(w.st_text, emb, (size_t)batch * DTXT * 4, cudaMemcpyDefault, st));
  KD_TRY(launch(c, CLS_SETUP, 0, (double)batch * DTXT * 6, st, "pack_embeddings", [&] {
    return pack_embeddings(w.st_text, batch, nullptr, 1, 0, w.emb, c->bf16(), st);
  }));
  KD_TRY(timestep_rows(c, t, 0, 1, st));
  KD_TRY(condition_setup(c, net, batch, 1, st));
  void* A = net == 0 ? w.A_root : w.A_body;
  const int lda = net == 0 ? ROOT_IN_LD : BODY_IN_LD;
  KD_TRY(launch(c, CLS_MOTION, 0, (double)batch * frames * n.din * 8, st, "pack_frames", [&] {
    return pack_frames(w.x, batch, n.din, 0, n.din, A, c->bf16(), lda, 0, batch, frames, frames + 1, st);
  }));
  float* hat = net == 0 ? w.root_hat : w.body_hat;
  KD_TRY(run_net(c, net, batch, frames, batch, A, w.tmlp[net], w.txt[net], hat, st));
  KD_CUDA(cudaMemcpyAsync(out, hat, (size_t)batch * frames * n.dout * 4, cudaMemcpyDefault, st));
  c->last_launches = c->launches - l0;
  return finish_outputs(c, out, st);
}
