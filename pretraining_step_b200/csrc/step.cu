// step.cu -- the step driver behind the C ABI: parameter / gradient /
// activation storage, the forward + backward sequence of the depth-L GPT,
// the Muon step, and the op-level entry points.
//
// Model (dev.to guide "Como treinar seu proprio ChatGPT por 50 dolares",
// section "1. Modelo GPT"):  x0 = wte[tok];  per layer
//   h1 = rms(x);  [q k v] = h1 [wq wk wv]^T;  q, k <- rms_head(rope(.));
//   o = causal_attention(q, k, v);  x <- x + o wo^T;
// (k and v have Hkv heads, query head h reading KV head h / (H / Hkv); a
// layer may attend through a causal left window: the guide's fewer KV heads
// and short/long window pattern.  The default is Hkv = H, no windows.)
//   h2 = rms(x);  a = relu(h2 wup^T)^2;  x <- x + a wdown^T;
// then z = rms(x) lm_head^T and loss = mean(lse(z) - z[target]).
// Residual stream and every row statistic are fp32; GEMM operands are bf16
// with fp32 accumulation in TMEM.
//
// Memory layout in HBM (one allocation per role):
//   wte [V,d] f32;  blocks [L][10 d^2 + 2 dkv d] f32 masters + bf16 copies
//   (dkv = 128 Hkv; = d by default, 12 d^2 per layer): wq [d,d] | wk [dkv,d]
//   | wv [dkv,d] (one [d + 2 dkv, d] matrix) | wo [d,d] | wup [4d,d] |
//   wdown [d,4d];
//   lm_head [V,d] f32 + bf16;  Muon momentum like blocks (f32).
//   Activations per B*T tokens: x_0..x_L and the mid-layer residuals (f32),
//   h1, h2, qkv, o, a (bf16), row statistics (f32), logits [N,V] bf16
//   (overwritten in place by their gradient), backward scratch.

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace nc {

// ------------------------------------------------------------------ errors
static thread_local std::string g_last_error;
void set_error(const std::string& msg) { g_last_error = msg; }
nc_status fail(nc_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}
nc_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return e == cudaErrorMemoryAllocation ? NC_ERR_OOM : NC_ERR_CUDA;
}

int num_sms() {
  static int n = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  });
  return n;
}

namespace {

typedef __nv_bfloat16 bf16;

// Bump allocator over one cudaMalloc.
struct Arena {
  char* base = nullptr;
  size_t size = 0, used = 0;
  template <class T>
  T* take(int64_t n) {
    const size_t bytes = ((size_t)n * sizeof(T) + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base + used);
    used += bytes;
    return p;
  }
};

struct Acts {
  int64_t N = 0;
  int B = 0, T = 0;
  void* mem = nullptr;
  int32_t *tok = nullptr, *tgt = nullptr;
  std::vector<float*> x, xmid, r1, r2, rq, rk, lse;
  std::vector<bf16*> h1, h2, qkv, o, a;
  bf16 *hf = nullptr, *logits = nullptr, *dxb = nullptr, *dh = nullptr, *du = nullptr,
       *dqkv = nullptr, *ds = nullptr;
  int64_t ld_ds = 0;  // row stride of ds: T rounded up to a multiple of 8
  float *rf = nullptr, *loss_rows = nullptr, *loss = nullptr, *dx0 = nullptr, *dx1 = nullptr,
        *delta = nullptr;
  // fp8 mode: E4M3 copies of the forward activations each layer's
  // projections read, in both layouts (K-major for the forward GEMM, the
  // transpose for the weight gradient's): q8f[l][0..7] = h1, h1^T, o, o^T,
  // h2, h2^T, a, a^T.  q8g / q8gT: the gradient being propagated, both
  // layouts; q8w: one weight (or its transpose).  f8sc[l][g][2]: the (A, B)
  // scales of GEMM g of layer l (F8_*); f8scratch: amax scratch.
  std::vector<std::array<uint8_t*, 8>> q8f;
  uint8_t *q8g = nullptr, *q8gT = nullptr, *q8w = nullptr;
  float* f8sc = nullptr;
  unsigned* f8scratch = nullptr;
};

// The twelve E4M3 GEMMs of a layer in fp8 mode (their scale pairs in f8sc).
enum { F8_QKV_F, F8_O_F, F8_UP_F, F8_DOWN_F, F8_QKV_D, F8_O_D, F8_UP_D, F8_DOWN_D,
       F8_QKV_W, F8_O_W, F8_UP_W, F8_DOWN_W, F8_COUNT };

}  // namespace
}  // namespace nc

struct nc_params {
  int depth = 0, vocab = 0, d = 0, H = 0, hd = 0, F = 0;
  int Hkv = 0, dkv = 0;     // KV heads and the width of k, v (dkv = 128 Hkv)
  bool fp8 = false;         // block projections on E4M3 operands
  // The weight-gradient GEMMs of the bf16 backward run on a second stream
  // (wg), forked from and joined to the step's stream by events: fork[k]
  // when the GEMM's inputs are ready, done[k] once it has read them.
  cudaStream_t wg = nullptr;
  cudaEvent_t wg_fork[4] = {}, wg_done[4] = {};
  int64_t lm_chunk = 32768;  // tokens per lm_head + cross-entropy chunk
  std::vector<int> window;  // per layer: causal left window, -1 = full causal
  cudaStream_t stream = nullptr;
  nc::Profiler* prof = nullptr;
  int* status = nullptr;  // device status word
  bool poisoned = false;
  void* pmem = nullptr;
  float *wte = nullptr, *blocks = nullptr, *lm = nullptr, *mom = nullptr;
  nc::bf16 *blocks_b = nullptr, *lm_b = nullptr;
  // Muon
  float* sumsq = nullptr;
  nc::bf16 *xsq = nullptr, *xw = nullptr, *nsws = nullptr;
  nc::bf16* xkv = nullptr;  // wk, wv stack when dkv < d (their own Newton-Schulz shape)
  // AdamW state of wte and lm_head (first and second moments, allocated
  // and zeroed by the first nc_adamw_step) and the step count
  float* adam = nullptr;
  int adam_t = 0;
  // RoPE table
  float2* rope = nullptr;
  int rope_T = 0;
  nc::Acts act;
  // pinned host staging for loss + status
  float* h_loss = nullptr;
  int* h_status = nullptr;
  // One captured step (nc_step_capture) and its kernel launches per replay.
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t graph_exec = nullptr;
  int64_t graph_launches = 0;
  const nc_grads* graph_g = nullptr;  // the gradients the captured step writes
};

struct nc_grads {
  const nc_params* p = nullptr;
  void* mem = nullptr;
  float *wte = nullptr, *blocks = nullptr, *lm = nullptr;
};

namespace nc {
namespace {

// Elements of one layer's block matrices and the offset of matrix j
// (0..5: wq, wk, wv, wo, wup, wdown) inside it.
int64_t layer_elems(const nc_params* p) {
  return 10ll * p->d * p->d + 2ll * p->dkv * p->d;
}
int64_t mat_offset(const nc_params* p, int j) {
  const int64_t d2 = (int64_t)p->d * p->d, kv = (int64_t)p->dkv * p->d;
  switch (j) {
    case 0: return 0;
    case 1: return d2;
    case 2: return d2 + kv;
    case 3: return d2 + 2 * kv;
    case 4: return 2 * d2 + 2 * kv;
    default: return 6 * d2 + 2 * kv;
  }
}
int64_t block_elems(const nc_params* p) { return p->depth * layer_elems(p); }
int64_t qkv_width(const nc_params* p) { return (int64_t)p->d + 2ll * p->dkv; }

// Offset and shape of parameter tensor idx (interface order).
void tensor_layout(const nc_params* p, int idx, int64_t* off, int64_t* rows, int64_t* cols,
                   const char** name, int* layer) {
  const int64_t d = p->d;
  const int n = 6 * p->depth + 2;
  *layer = -1;
  if (idx == 0) {
    *off = 0; *rows = p->vocab; *cols = d; *name = "wte";
  } else if (idx == n - 1) {
    *off = 0; *rows = p->vocab; *cols = d; *name = "lm_head";
  } else {
    const int l = (idx - 1) / 6, j = (idx - 1) % 6;
    static const char* names[6] = {"wq", "wk", "wv", "wo", "wup", "wdown"};
    *layer = l;
    *name = names[j];
    *off = l * layer_elems(p) + mat_offset(p, j);
    *rows = (j == 4) ? 4 * d : (j == 1 || j == 2) ? p->dkv : d;
    *cols = (j == 5) ? 4 * d : d;
  }
}

nc_status check_status(nc_params* p) {
  // Called after a synchronisation that copied the status word.
  const int st = *p->h_status;
  if (st == kDevOk) return NC_OK;
  if (st == kDevTimeout) {
    p->poisoned = true;
    return fail(NC_ERR_TIMEOUT, "a device wait timed out; the handle is poisoned");
  }
  if (st == kDevTokenRange) return fail(NC_ERR_TOKEN_RANGE, "token or target id out of [0, vocab)");
  return fail(NC_ERR_CUDA, "unknown device status");
}

nc_status sync_and_check(nc_params* p, const float* loss_dev) {
  if (loss_dev)
    NC_CUDA_TRY(cudaMemcpyAsync(p->h_loss, loss_dev, sizeof(float), cudaMemcpyDeviceToHost,
                                p->stream));
  NC_CUDA_TRY(cudaMemcpyAsync(p->h_status, p->status, sizeof(int), cudaMemcpyDeviceToHost,
                              p->stream));
  NC_CUDA_TRY(cudaStreamSynchronize(p->stream));
  nc_status s = check_status(p);
  if (*p->h_status == kDevTokenRange) {
    NC_CUDA_TRY(cudaMemsetAsync(p->status, 0, sizeof(int), p->stream));
    NC_CUDA_TRY(cudaStreamSynchronize(p->stream));
  }
  return s;
}

// A captured step holds the addresses of the activations and the RoPE
// table: it is released before either is reallocated.
void drop_graph(nc_params* p) {
  if (p->graph_exec) cudaGraphExecDestroy(p->graph_exec);
  if (p->graph) cudaGraphDestroy(p->graph);
  p->graph_exec = nullptr;
  p->graph = nullptr;
  p->graph_launches = 0;
  p->graph_g = nullptr;
}

nc_status ensure_rope(nc_params* p, int T) {
  if (p->rope_T >= T) return NC_OK;
  drop_graph(p);
  int newT = std::max(T, 2048);
  if (p->rope) cudaFree(p->rope);
  p->rope = nullptr;
  NC_CUDA_TRY(cudaMalloc(&p->rope, 2 * sizeof(float2) * (size_t)newT * (p->hd / 2)));  // two layouts
  NC_TRY(rope_table(p->rope, newT, p->hd, p->stream));
  p->rope_T = newT;
  return NC_OK;
}

nc_status ensure_acts(nc_params* p, int B, int T) {
  Acts& a = p->act;
  const int64_t N = (int64_t)B * T;
  if (a.mem && a.N == N && a.B == B && a.T == T) return NC_OK;
  if (a.mem) {
    NC_CUDA_TRY(cudaStreamSynchronize(p->stream));
    drop_graph(p);
    cudaFree(a.mem);
    a = Acts();
  }
  const int L = p->depth;
  const int64_t d = p->d, F = p->F, V = p->vocab, H = p->H, Hkv = p->Hkv, Q = qkv_width(p);
  // Sizes in bytes, each rounded to 256.
  auto r = [](int64_t bytes) { return (bytes + 255) & ~int64_t(255); };
  int64_t total = 0;
  total += 2 * r(4 * N);                                     // tok, tgt
  total += (L + 1) * r(4 * N * d) + L * r(4 * N * d);        // x, xmid
  total += 2 * L * r(4 * N) + L * r(4 * N * H) + L * r(4 * N * Hkv);  // r1 r2 rq rk
  total += L * r(4 * N * H);                                 // lse [B,H,T]
  total += 2 * L * r(2 * N * d) + L * r(2 * N * Q) + L * r(2 * N * d) + L * r(2 * N * F);
  const int64_t NC = std::min<int64_t>(p->lm_chunk, N);  // logits rows held
  total += r(2 * N * d) + r(4 * N) + r(2 * NC * V) + r(4 * N) + r(4);  // hf rf logits loss
  const int64_t ld_ds = (T + 7) & ~int64_t(7);
  total += 2 * r(4 * N * d) + 2 * r(2 * N * d) + r(2 * N * F) + r(2 * N * Q) +
           r(4 * N * H);                                     // backward scratch
  total += r(2 * (int64_t)B * H * T * ld_ds);                // attention dS^T tiles
  const int64_t wmax = std::max(F, Q) * d;                   // largest weight, elements
  if (p->fp8)  // E4M3 operands: saved activations, the propagated gradient, a weight, scales
    total += L * (6 * r(N * d) + 2 * r(N * F)) + 2 * r(N * std::max(F, Q)) + r(wmax) +
             r(4 * L * F8_COUNT * 2) + r(8);
  void* mem = nullptr;
  cudaError_t e = cudaMalloc(&mem, (size_t)total);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(NC_ERR_OOM, "activation allocation of " + std::to_string(total >> 20) + " MiB failed");
  }
  Arena ar{static_cast<char*>(mem), (size_t)total, 0};
  a.mem = mem;
  a.N = N;
  a.B = B;
  a.T = T;
  a.tok = ar.take<int32_t>(N);
  a.tgt = ar.take<int32_t>(N);
  for (int l = 0; l <= L; ++l) a.x.push_back(ar.take<float>(N * d));
  for (int l = 0; l < L; ++l) {
    a.xmid.push_back(ar.take<float>(N * d));
    a.r1.push_back(ar.take<float>(N));
    a.r2.push_back(ar.take<float>(N));
    a.rq.push_back(ar.take<float>(N * H));
    a.rk.push_back(ar.take<float>(N * Hkv));
    a.lse.push_back(ar.take<float>(N * H));
    a.h1.push_back(ar.take<bf16>(N * d));
    a.h2.push_back(ar.take<bf16>(N * d));
    a.qkv.push_back(ar.take<bf16>(N * Q));
    a.o.push_back(ar.take<bf16>(N * d));
    a.a.push_back(ar.take<bf16>(N * F));
  }
  a.hf = ar.take<bf16>(N * d);
  a.rf = ar.take<float>(N);
  a.logits = ar.take<bf16>(NC * V);
  a.loss_rows = ar.take<float>(N);
  a.loss = ar.take<float>(1);
  a.dx0 = ar.take<float>(N * d);
  a.dx1 = ar.take<float>(N * d);
  a.dxb = ar.take<bf16>(N * d);
  a.dh = ar.take<bf16>(N * d);
  a.du = ar.take<bf16>(N * F);
  a.dqkv = ar.take<bf16>(N * Q);
  a.delta = ar.take<float>(N * H);
  a.ld_ds = ld_ds;
  a.ds = ar.take<bf16>((int64_t)B * H * T * ld_ds);
  if (p->fp8) {
    a.q8f.resize(L);
    for (int l = 0; l < L; ++l)
      for (int j = 0; j < 8; ++j) a.q8f[l][j] = ar.take<uint8_t>(j < 6 ? N * d : N * F);
    a.q8g = ar.take<uint8_t>(N * std::max(F, Q));
    a.q8gT = ar.take<uint8_t>(N * std::max(F, Q));
    a.q8w = ar.take<uint8_t>(wmax);
    a.f8sc = ar.take<float>((int64_t)L * F8_COUNT * 2);
    a.f8scratch = ar.take<unsigned>(2);  // [0] amax computed by the quantiser, [1] by a GEMM epilogue
  }
  if (ar.used > ar.size) return fail(NC_ERR_CUDA, "activation arena overflow");
  return NC_OK;
}

bool is_device_ptr(const void* ptr) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

// fp8 mode: the fp32 master of a block matrix from its bf16 copy.
const float* master_of(const nc_params* p, const bf16* Wb) { return p->blocks + (Wb - p->blocks_b); }

// fp8 mode: an activation or gradient (bf16 [rows, cols], row stride ld) to
// E4M3 in both layouts (either may be null), its scale to s0 (and s1).
// amax: the word where the tensor's producer folded in max |x| (zeroed
// before it ran), or null to compute it here.
nc_status quant8(nc_params* p, const bf16* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* q,
                 uint8_t* qT, float* s0, float* s1, unsigned* amax = nullptr) {
  return fp8_quantize2(x, rows, (int)cols, ld, q, qT, s0, s1, amax ? amax : p->act.f8scratch, amax != nullptr,
                       p->stream, p->prof);
}

// fp8 mode: the fp32 master of a block matrix ([rows, cols]) to E4M3 in
// p->act.q8w, as is or transposed, its scale to s.
nc_status quant8w(nc_params* p, const bf16* Wb, int64_t rows, int64_t cols, bool transpose, float* s) {
  return fp8_quantize(master_of(p, Wb), false, rows, (int)cols, cols, transpose, p->act.q8w,
                      transpose ? rows : cols, s, p->act.f8scratch, p->stream, p->prof);
}

// fp8 mode: the word (zeroed here) a norm or GEMM epilogue folds its bf16
// output's amax into, for that output's quantisation; null in bf16 mode.
nc_status amax_word(nc_params* p, unsigned** w) {
  *w = nullptr;
  if (!p->fp8) return NC_OK;
  *w = p->act.f8scratch + 1;
  NC_CUDA_TRY(cudaMemsetAsync(*w, 0, sizeof(unsigned), p->stream));
  return NC_OK;
}

// One E4M3 GEMM: D[M, N] = epi(A8[M, K] B8[N, K]^T / (sc[0] sc[1])), both
// operands K-major; weight gradients (NC_EPI_ACC_F32) split K automatically.
nc_status gemm8(nc_params* p, int64_t M, int64_t N, int64_t K, const uint8_t* A8, int64_t lda,
                const uint8_t* B8, int64_t ldb, void* D, int64_t ldd, nc_epilogue epi, const void* aux,
                int64_t ldaux, const float* sc, const char* tag, unsigned* amax_out = nullptr) {
  GemmLaunch g{};
  g.status = p->status;
  g.tag = tag;
  g.d.M = (int)M; g.d.N = (int)N; g.d.K = (int)K; g.d.batch = 1;
  g.d.A = A8; g.d.lda = lda; g.d.a_kmajor = 1;
  g.d.B = B8; g.d.ldb = ldb; g.d.b_kmajor = 1;
  g.d.D = D; g.d.ldd = ldd;
  g.d.aux = aux; g.d.ldaux = ldaux;
  g.d.epi = epi; g.d.alpha = 1.f; g.d.split_k = epi == NC_EPI_ACC_F32 ? 0 : 1;
  g.d.ab_type = 1;
  g.d.ab_scale = sc;
  g.d.amax_out = amax_out;
  if (amax_out) NC_CUDA_TRY(cudaMemsetAsync(amax_out, 0, sizeof(unsigned), p->stream));
  return gemm_launch(g, p->stream, p->prof);
}

// y[M,N] = epi(x[M,K] W[N,K]^T): the forward projection.
nc_status proj(nc_params* p, const bf16* x, int64_t M, int64_t K, const bf16* W, int64_t Nout,
               void* D, int64_t ldd, nc_epilogue epi, const void* aux, int64_t ldaux,
               const char* tag = "gemm_fwd") {
  GemmLaunch g{};
  g.status = p->status;
  g.tag = tag;
  g.d.M = (int)M; g.d.N = (int)Nout; g.d.K = (int)K; g.d.batch = 1;
  g.d.A = x; g.d.lda = K; g.d.a_kmajor = 1;
  g.d.B = W; g.d.ldb = K; g.d.b_kmajor = 1;
  g.d.D = D; g.d.ldd = ldd;
  g.d.aux = aux; g.d.ldaux = ldaux;
  g.d.epi = epi; g.d.alpha = 1.f; g.d.split_k = 1;
  return gemm_launch(g, p->stream, p->prof);
}

// dx[M,N] = epi(dy[M,K] W[K,N]): the input gradient of a projection.
nc_status proj_dx(nc_params* p, const bf16* dy, int64_t M, int64_t K, const bf16* W, int64_t Nout,
                  void* D, int64_t ldd, nc_epilogue epi, const void* aux, int64_t ldaux,
                  const char* tag = "gemm_dgrad") {
  GemmLaunch g{};
  g.status = p->status;
  g.tag = tag;
  g.d.M = (int)M; g.d.N = (int)Nout; g.d.K = (int)K; g.d.batch = 1;
  g.d.A = dy; g.d.lda = K; g.d.a_kmajor = 1;
  g.d.B = W; g.d.ldb = Nout; g.d.b_kmajor = 0;
  g.d.D = D; g.d.ldd = ldd;
  g.d.aux = aux; g.d.ldaux = ldaux;
  g.d.epi = epi; g.d.alpha = 1.f; g.d.split_k = 1;
  return gemm_launch(g, p->stream, p->prof);
}

// dW[Mo,No] = dy[Ntok,Mo]^T x[Ntok,No] into a zeroed fp32 gradient.
nc_status proj_dw(nc_params* p, const bf16* dy, int64_t ldy, int64_t Mo, const bf16* x,
                  int64_t ldx, int64_t No, int64_t Ntok, float* dW,
                  const char* tag = "gemm_wgrad", cudaStream_t st = nullptr) {
  GemmLaunch g{};
  g.status = p->status;
  g.tag = tag;
  g.d.M = (int)Mo; g.d.N = (int)No; g.d.K = (int)Ntok; g.d.batch = 1;
  g.d.A = dy; g.d.lda = ldy; g.d.a_kmajor = 0;
  g.d.B = x; g.d.ldb = ldx; g.d.b_kmajor = 0;
  g.d.D = dW; g.d.ldd = No;
  g.d.epi = NC_EPI_ACC_F32; g.d.alpha = 1.f; g.d.split_k = 0;  // automatic split
  return gemm_launch(g, st ? st : p->stream, p->prof);
}

// The backward of layer l in fp8 mode: the layer's eight GEMMs on E4M3
// operands (the propagated gradient quantised once per projection in both
// layouts, the forward activations' transposes saved by the forward, each
// weight's transpose from its master), the rest as in the bf16 step.  dx:
// the residual gradient, in and out (through dxn, as the bf16 step's two
// norm backwards do); a.dxb its bf16 copy.
nc_status layer_bwd_fp8(nc_params* p, int l, int B, int T, const bf16* W, float* G, float* dx, float* dxn) {
  Acts& a = p->act;
  cudaStream_t s = p->stream;
  Profiler* pr = p->prof;
  const int H = p->H, Hkv = p->Hkv;
  const int64_t N = (int64_t)B * T, d = p->d, F = p->F, dkv = p->dkv, Q = qkv_width(p);
  const int64_t o_wo = mat_offset(p, 3), o_up = mat_offset(p, 4), o_down = mat_offset(p, 5);
  float* sc = a.f8sc + ((int64_t)l * F8_COUNT) * 2;
  auto& q = a.q8f[l];
  // MLP: x_out = xmid + a wdown^T, a = relu(h2 wup^T)^2 (dxb's amax from the norm that wrote it)
  NC_TRY(quant8(p, a.dxb, N, d, d, a.q8g, a.q8gT, sc + 2 * F8_DOWN_D, sc + 2 * F8_DOWN_W, a.f8scratch + 1));
  NC_TRY(gemm8(p, d, F, N, a.q8gT, N, q[7], N, G + o_down, F, NC_EPI_ACC_F32, nullptr, 0, sc + 2 * F8_DOWN_W,
               "gemm_wgrad"));
  NC_TRY(quant8w(p, W + o_down, d, F, true, sc + 2 * F8_DOWN_D + 1));
  NC_TRY(gemm8(p, N, F, d, a.q8g, d, a.q8w, d, a.du, F, NC_EPI_RELU2_BWD, a.a[l], F, sc + 2 * F8_DOWN_D,
               "gemm_dgrad", a.f8scratch + 1));
  NC_TRY(quant8(p, a.du, N, F, F, a.q8g, a.q8gT, sc + 2 * F8_UP_D, sc + 2 * F8_UP_W, a.f8scratch + 1));
  NC_TRY(gemm8(p, F, d, N, a.q8gT, N, q[5], N, G + o_up, d, NC_EPI_ACC_F32, nullptr, 0, sc + 2 * F8_UP_W,
               "gemm_wgrad"));
  NC_TRY(quant8w(p, W + o_up, F, d, true, sc + 2 * F8_UP_D + 1));
  NC_TRY(gemm8(p, N, d, F, a.q8g, F, a.q8w, F, a.dh, d, NC_EPI_STORE_BF16, nullptr, 0, sc + 2 * F8_UP_D,
               "gemm_dgrad"));
  unsigned* am = nullptr;
  NC_TRY(amax_word(p, &am));
  NC_TRY(rmsnorm_bwd(a.dh, a.h2[l], a.r2[l], dx, N, (int)d, dxn, a.dxb, s, pr, am));
  std::swap(dx, dxn);
  // Attention: xmid = x + o wo^T
  NC_TRY(quant8(p, a.dxb, N, d, d, a.q8g, a.q8gT, sc + 2 * F8_O_D, sc + 2 * F8_O_W, am));
  NC_TRY(gemm8(p, d, d, N, a.q8gT, N, q[3], N, G + o_wo, d, NC_EPI_ACC_F32, nullptr, 0, sc + 2 * F8_O_W,
               "gemm_wgrad"));
  NC_TRY(quant8w(p, W + o_wo, d, d, true, sc + 2 * F8_O_D + 1));
  NC_TRY(gemm8(p, N, d, d, a.q8g, d, a.q8w, d, a.dh, d, NC_EPI_STORE_BF16, nullptr, 0, sc + 2 * F8_O_D,
               "gemm_dgrad"));
  NC_TRY(attention_bwd_model(a.qkv[l], Q, a.qkv[l] + d, a.qkv[l] + d + dkv, Q, a.o[l], a.dh, d, a.lse[l],
                             a.delta, a.ds, a.ld_ds, a.dqkv, a.dqkv + d, a.dqkv + d + dkv, Q, B, T, H, Hkv,
                             p->window[l], p->rope, p->rope_T, a.rq[l], a.rk[l], p->status, s, pr));
  NC_TRY(quant8(p, a.dqkv, N, Q, Q, a.q8g, a.q8gT, sc + 2 * F8_QKV_D, sc + 2 * F8_QKV_W));
  NC_TRY(gemm8(p, Q, d, N, a.q8gT, N, q[1], N, G, d, NC_EPI_ACC_F32, nullptr, 0, sc + 2 * F8_QKV_W,
               "gemm_wgrad"));
  NC_TRY(quant8w(p, W, Q, d, true, sc + 2 * F8_QKV_D + 1));
  NC_TRY(gemm8(p, N, d, Q, a.q8g, Q, a.q8w, Q, a.dh, d, NC_EPI_STORE_BF16, nullptr, 0, sc + 2 * F8_QKV_D,
               "gemm_dgrad"));
  // Back into the caller's dx (dxn here, after the swap above); its amax
  // for the next layer's first quantisation.
  NC_TRY(amax_word(p, &am));
  NC_TRY(rmsnorm_bwd(a.dh, a.h1[l], a.r1[l], dx, N, (int)d, dxn, a.dxb, s, pr, am));
  return NC_OK;
}

// ids_on_device: the caller has established that tokens and targets are
// device memory (a graph capture, which records no pointer queries).
nc_status fwd_bwd(nc_params* p, const int32_t* tokens, const int32_t* targets, int B, int T,
                  float* loss_dev, nc_grads* g, bool ids_on_device = false) {
  if (p->poisoned) return fail(NC_ERR_TIMEOUT, "handle poisoned by an earlier device timeout");
  if (!tokens || !targets || !g || g->p != p || B < 1 || T < 1 || (int64_t)B * T > (1 << 24))
    return fail(NC_ERR_INVALID_ARG, "fwd_bwd: bad arguments");
  if (p->fp8 && (((int64_t)B * T) % 16 || (int64_t)B * T <= 128))
    return fail(NC_ERR_INVALID_ARG, "fwd_bwd: fp8 mode needs B*T > 128 and a multiple of 16");
  NC_TRY(ensure_acts(p, B, T));
  NC_TRY(ensure_rope(p, T));
  Acts& a = p->act;
  cudaStream_t s = p->stream;
  Profiler* pr = p->prof;
  const int L = p->depth, H = p->H, Hkv = p->Hkv, hd = p->hd, V = p->vocab;
  const int64_t N = (int64_t)B * T, d = p->d, F = p->F, dkv = p->dkv, Q = qkv_width(p);
  const int64_t LS = layer_elems(p);
  const int64_t o_wo = mat_offset(p, 3), o_up = mat_offset(p, 4), o_down = mat_offset(p, 5);

  const int32_t* tok = tokens;
  const int32_t* tgt = targets;
  if (!ids_on_device && !is_device_ptr(tokens)) {
    NC_CUDA_TRY(cudaMemcpyAsync(a.tok, tokens, 4 * N, cudaMemcpyHostToDevice, s));
    tok = a.tok;
  }
  if (!ids_on_device && !is_device_ptr(targets)) {
    NC_CUDA_TRY(cudaMemcpyAsync(a.tgt, targets, 4 * N, cudaMemcpyHostToDevice, s));
    tgt = a.tgt;
  }
  NC_CUDA_TRY(cudaMemsetAsync(g->mem, 0, sizeof(float) * (2 * (int64_t)V * d + block_elems(p)), s));

  // ---------------- forward
  NC_TRY(embed_gather(tok, N, p->wte, V, (int)d, a.x[0], p->status, s, pr));
  for (int l = 0; l < L; ++l) {
    const bf16* W = p->blocks_b + l * LS;
    unsigned* am = nullptr;
    NC_TRY(amax_word(p, &am));
    NC_TRY(rmsnorm_fwd(a.x[l], N, (int)d, a.h1[l], a.r1[l], s, pr, am));
    {
      // q|k|v projection with RoPE + QK-norm fused into the epilogue.
      GemmLaunch g{};
      g.status = p->status;
      g.tag = "gemm_fwd";
      g.d.M = (int)N; g.d.N = (int)Q; g.d.K = (int)d; g.d.batch = 1;
      g.d.A = a.h1[l]; g.d.lda = d; g.d.a_kmajor = 1;
      g.d.B = W; g.d.ldb = d; g.d.b_kmajor = 1;
      g.d.D = a.qkv[l]; g.d.ldd = Q;
      g.d.epi = NC_EPI_ROPE_QKNORM; g.d.alpha = 1.f; g.d.split_k = 1;
      g.d.rope_T = T; g.d.rope_H = H; g.d.rope_Hkv = Hkv; g.d.rope_tab = p->rope;
      g.d.rstd_q = a.rq[l]; g.d.rstd_k = a.rk[l];
      if (p->fp8) {  // h1 in both layouts (the transpose for the weight gradient); wq|wk|wv as one tensor
        float* sc = a.f8sc + ((int64_t)l * F8_COUNT) * 2;
        NC_TRY(quant8(p, a.h1[l], N, d, d, a.q8f[l][0], a.q8f[l][1], sc + 2 * F8_QKV_F, sc + 2 * F8_QKV_W + 1,
                      am));
        NC_TRY(quant8w(p, W, Q, d, false, sc + 2 * F8_QKV_F + 1));
        g.d.A = a.q8f[l][0]; g.d.lda = d;
        g.d.B = a.q8w; g.d.ldb = d;
        g.d.ab_type = 1;
        g.d.ab_scale = sc + 2 * F8_QKV_F;
      }
      NC_TRY(gemm_launch(g, s, pr));
    }
    NC_TRY(attention_fwd_ex(a.qkv[l], Q, a.qkv[l] + d, a.qkv[l] + d + dkv, Q, a.o[l], d,
                            a.lse[l], B, T, H, Hkv, p->window[l], p->status, s, pr));
    if (p->fp8) {
      float* sc = a.f8sc + ((int64_t)l * F8_COUNT) * 2;
      auto& q = a.q8f[l];
      NC_TRY(quant8(p, a.o[l], N, d, d, q[2], q[3], sc + 2 * F8_O_F, sc + 2 * F8_O_W + 1));
      NC_TRY(quant8w(p, W + o_wo, d, d, false, sc + 2 * F8_O_F + 1));
      NC_TRY(gemm8(p, N, d, d, q[2], d, a.q8w, d, a.xmid[l], d, NC_EPI_RESID_F32, a.x[l], d,
                   sc + 2 * F8_O_F, "gemm_fwd"));
      NC_TRY(amax_word(p, &am));
      NC_TRY(rmsnorm_fwd(a.xmid[l], N, (int)d, a.h2[l], a.r2[l], s, pr, am));
      NC_TRY(quant8(p, a.h2[l], N, d, d, q[4], q[5], sc + 2 * F8_UP_F, sc + 2 * F8_UP_W + 1, am));
      NC_TRY(quant8w(p, W + o_up, F, d, false, sc + 2 * F8_UP_F + 1));
      NC_TRY(gemm8(p, N, F, d, q[4], d, a.q8w, d, a.a[l], F, NC_EPI_RELU2, nullptr, 0, sc + 2 * F8_UP_F,
                   "gemm_fwd", a.f8scratch + 1));
      NC_TRY(quant8(p, a.a[l], N, F, F, q[6], q[7], sc + 2 * F8_DOWN_F, sc + 2 * F8_DOWN_W + 1,
                    a.f8scratch + 1));
      NC_TRY(quant8w(p, W + o_down, d, F, false, sc + 2 * F8_DOWN_F + 1));
      NC_TRY(gemm8(p, N, d, F, q[6], F, a.q8w, F, a.x[l + 1], d, NC_EPI_RESID_F32, a.xmid[l], d,
                   sc + 2 * F8_DOWN_F, "gemm_fwd"));
      continue;
    }
    NC_TRY(proj(p, a.o[l], N, d, W + o_wo, d, a.xmid[l], d, NC_EPI_RESID_F32, a.x[l], d));
    NC_TRY(rmsnorm_fwd(a.xmid[l], N, (int)d, a.h2[l], a.r2[l], s, pr));
    NC_TRY(proj(p, a.h2[l], N, d, W + o_up, F, a.a[l], F, NC_EPI_RELU2, nullptr, 0));
    NC_TRY(proj(p, a.a[l], N, F, W + o_down, d, a.x[l + 1], d, NC_EPI_RESID_F32, a.xmid[l], d));
  }
  NC_TRY(rmsnorm_fwd(a.x[L], N, (int)d, a.hf, a.rf, s, pr));
  // lm_head + cross-entropy in chunks of lm_chunk tokens: logits of the
  // chunk, its loss rows and, in place, its dz
  // (scaled by 1 / N of the whole batch); then dW_lm += dz^T hf and dh = dz
  // W_lm for the chunk's rows, so only one chunk's logits are ever held.
  {
    const int64_t NC = std::min<int64_t>(p->lm_chunk, N);
    for (int64_t c0 = 0; c0 < N; c0 += NC) {
      const int64_t nc = std::min(NC, N - c0);
      NC_TRY(proj(p, a.hf + c0 * d, nc, d, p->lm_b, V, a.logits, V, NC_EPI_STORE_BF16, nullptr, 0,
                  "gemm_lmhead"));
      NC_TRY(ce_fwd_bwd(a.logits, tgt + c0, nc, V, 1.0f / (float)N, a.loss_rows + c0, p->status, s, pr));
      NC_TRY(proj_dw(p, a.logits, V, V, a.hf + c0 * d, d, d, nc, g->lm, "gemm_lmhead"));
      NC_TRY(proj_dx(p, a.logits, nc, V, p->lm_b, d, a.dh + c0 * d, d, NC_EPI_STORE_BF16, nullptr, 0,
                     "gemm_lmhead"));
    }
    NC_TRY(loss_mean(a.loss_rows, N, loss_dev ? loss_dev : a.loss, s));
  }
  float* dx = a.dx0;
  float* dxn = a.dx1;
  {
    unsigned* am = nullptr;  // fp8: dxb's amax for the last layer's first quantisation
    NC_TRY(amax_word(p, &am));
    NC_TRY(rmsnorm_bwd(a.dh, a.hf, a.rf, nullptr, N, (int)d, dx, a.dxb, s, pr, am));
  }
  const bool two_streams = !p->fp8 && !profiler_enabled(pr);
  for (int l = L - 1; l >= 0; --l) {
    const bf16* W = p->blocks_b + l * LS;
    float* G = g->blocks + l * LS;
    if (p->fp8) {
      NC_TRY(layer_bwd_fp8(p, l, B, T, W, G, dx, dxn));  // the gradient stays in dx
      continue;
    }
    // Each weight gradient goes to the wg stream as soon as its inputs are
    // ready; the step's stream waits for it only before it overwrites one
    // of them (dxb, du, dqkv).  wg work of the previous layer is ordered
    // before this layer's on wg itself.  While the per-launch profiler is
    // on, everything stays on the step's stream, so that each launch's
    // events time that launch alone.
    cudaStream_t w = two_streams ? p->wg : s;
    auto fork = [&](int k) -> nc_status {
      if (!two_streams) return NC_OK;
      NC_CUDA_TRY(cudaEventRecord(p->wg_fork[k], s));
      NC_CUDA_TRY(cudaStreamWaitEvent(w, p->wg_fork[k], 0));
      return NC_OK;
    };
    auto done = [&](int k) -> nc_status {
      if (!two_streams) return NC_OK;
      NC_CUDA_TRY(cudaEventRecord(p->wg_done[k], w));
      return NC_OK;
    };
    auto wait_done = [&](int k) -> nc_status {
      if (!two_streams) return NC_OK;
      NC_CUDA_TRY(cudaStreamWaitEvent(s, p->wg_done[k], 0));
      return NC_OK;
    };
    // MLP: x_out = xmid + a wdown^T, a = relu(h2 wup^T)^2
    NC_TRY(fork(0));
    NC_TRY(proj_dw(p, a.dxb, d, d, a.a[l], F, F, N, G + o_down, "gemm_wgrad", w));
    NC_TRY(done(0));
    if (l < L - 1) NC_TRY(wait_done(1));  // the previous layer's dW_up has read du
    NC_TRY(proj_dx(p, a.dxb, N, d, W + o_down, F, a.du, F, NC_EPI_RELU2_BWD, a.a[l], F));
    NC_TRY(fork(1));
    NC_TRY(proj_dw(p, a.du, F, F, a.h2[l], d, d, N, G + o_up, "gemm_wgrad", w));
    NC_TRY(done(1));
    NC_TRY(proj_dx(p, a.du, N, F, W + o_up, d, a.dh, d, NC_EPI_STORE_BF16, nullptr, 0));
    NC_TRY(wait_done(0));  // dW_down has read dxb
    NC_TRY(rmsnorm_bwd(a.dh, a.h2[l], a.r2[l], dx, N, (int)d, dxn, a.dxb, s, pr));
    std::swap(dx, dxn);
    // Attention: xmid = x + o wo^T
    NC_TRY(fork(2));
    NC_TRY(proj_dw(p, a.dxb, d, d, a.o[l], d, d, N, G + o_wo, "gemm_wgrad", w));
    NC_TRY(done(2));
    NC_TRY(proj_dx(p, a.dxb, N, d, W + o_wo, d, a.dh, d, NC_EPI_STORE_BF16, nullptr, 0));
    if (l < L - 1) NC_TRY(wait_done(3));  // the previous layer's dW_qkv has read dqkv
    // Key side (dK through the k-side RoPE + QK-norm backward, dV, dS^T to
    // a.ds), then the query side (dQ = dS K through the q-side backward).
    NC_TRY(attention_bwd_model(a.qkv[l], Q, a.qkv[l] + d, a.qkv[l] + d + dkv, Q, a.o[l], a.dh, d,
                               a.lse[l], a.delta, a.ds, a.ld_ds, a.dqkv, a.dqkv + d,
                               a.dqkv + d + dkv, Q, B, T, H, Hkv, p->window[l], p->rope, p->rope_T, a.rq[l],
                               a.rk[l], p->status, s, pr));
    NC_TRY(fork(3));
    NC_TRY(proj_dw(p, a.dqkv, Q, Q, a.h1[l], d, d, N, G, "gemm_wgrad", w));
    NC_TRY(done(3));
    NC_TRY(proj_dx(p, a.dqkv, N, Q, W, d, a.dh, d, NC_EPI_STORE_BF16, nullptr, 0));
    NC_TRY(wait_done(2));  // dW_o has read dxb
    NC_TRY(rmsnorm_bwd(a.dh, a.h1[l], a.r1[l], dx, N, (int)d, dxn, a.dxb, s, pr));
    std::swap(dx, dxn);
  }
  // Every weight gradient is complete before the step's stream goes on (the
  // optimiser reads them); wg's work is ordered, so its last event covers all.
  if (two_streams) NC_CUDA_TRY(cudaStreamWaitEvent(s, p->wg_done[3], 0));
  NC_TRY(embed_scatter(tok, N, dx, V, (int)d, g->wte, s, pr));
  return NC_OK;
}

nc_status muon(nc_params* p, const nc_grads* g, float lr, float mu) {
  if (p->poisoned) return fail(NC_ERR_TIMEOUT, "handle poisoned by an earlier device timeout");
  if (!g || g->p != p) return fail(NC_ERR_INVALID_ARG, "muon: gradients of another model");
  cudaStream_t s = p->stream;
  Profiler* pr = p->prof;
  const int L = p->depth;
  const int64_t d = p->d, d2 = d * d, dkv = p->dkv, kv = dkv * d, LS = layer_elems(p);
  NC_CUDA_TRY(cudaMemsetAsync(p->sumsq, 0, sizeof(float) * 6 * L, s));
  NC_TRY(muon_momentum(p->mom, g->blocks, L, (int)d, (int)dkv, mu, p->sumsq, s, pr));
  // Orthogonalisation stacks by shape: the d x d matrices (wq, wo, and wk, wv
  // when dkv = d) in xsq; wk, wv as dkv x d in xkv when dkv < d; wup
  // (transposed) and wdown as d x 4d in xw.  Stacks are [layer][matrix].
  const bool kv_square = dkv == d;
  const int n_sq = kv_square ? 4 : 2;
  const int sq_of[4] = {0, kv_square ? 1 : 3, 2, 3};
  for (int i = 0; i < n_sq; ++i)
    NC_TRY(muon_prep(p->mom + mat_offset(p, sq_of[i]), LS, (int)d, (int)d, 0, p->xsq + i * d2,
                     n_sq * d2, p->sumsq, sq_of[i], L, s, pr));
  if (!kv_square)
    for (int i = 0; i < 2; ++i)
      NC_TRY(muon_prep(p->mom + mat_offset(p, 1 + i), LS, (int)dkv, (int)d, 0, p->xkv + i * kv,
                       2 * kv, p->sumsq, 1 + i, L, s, pr));
  NC_TRY(muon_prep(p->mom + mat_offset(p, 4), LS, (int)(4 * d), (int)d, 1, p->xw, 8 * d2,
                   p->sumsq, 4, L, s, pr));
  NC_TRY(muon_prep(p->mom + mat_offset(p, 5), LS, (int)d, (int)(4 * d), 0, p->xw + 4 * d2, 8 * d2,
                   p->sumsq, 5, L, s, pr));
  NC_TRY(newton_schulz_wide(p->xsq, n_sq * L, (int)d, (int)d, 5, p->nsws, p->status, s, pr));
  if (!kv_square)
    NC_TRY(newton_schulz_wide(p->xkv, 2 * L, (int)dkv, (int)d, 5, p->nsws, p->status, s, pr));
  NC_TRY(newton_schulz_wide(p->xw, 2 * L, (int)d, (int)(4 * d), 5, p->nsws, p->status, s, pr));
  for (int i = 0; i < n_sq; ++i) {
    const int64_t o = mat_offset(p, sq_of[i]);
    NC_TRY(muon_apply(p->blocks + o, p->blocks_b + o, LS, (int)d, (int)d, 0, p->xsq + i * d2,
                      n_sq * d2, lr, L, s, pr));
  }
  if (!kv_square)
    for (int i = 0; i < 2; ++i) {
      const int64_t o = mat_offset(p, 1 + i);
      NC_TRY(muon_apply(p->blocks + o, p->blocks_b + o, LS, (int)dkv, (int)d, 0, p->xkv + i * kv,
                        2 * kv, lr, L, s, pr));
    }
  const int64_t o_up = mat_offset(p, 4), o_down = mat_offset(p, 5);
  NC_TRY(muon_apply(p->blocks + o_up, p->blocks_b + o_up, LS, (int)(4 * d), (int)d, 1, p->xw,
                    8 * d2, lr, L, s, pr));
  NC_TRY(muon_apply(p->blocks + o_down, p->blocks_b + o_down, LS, (int)d, (int)(4 * d), 0,
                    p->xw + 4 * d2, 8 * d2, lr, L, s, pr));
  return NC_OK;
}

nc_status sync_bf16(nc_params* p) {
  NC_TRY(f32_to_bf16(p->blocks, p->blocks_b, block_elems(p), p->stream, p->prof));
  NC_TRY(f32_to_bf16(p->lm, p->lm_b, (int64_t)p->vocab * p->d, p->stream, p->prof));
  return NC_OK;
}

uint64_t splitmix64_host(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

nc_status init_model(nc_params* p, uint64_t seed, int flags) {
  const int n = 6 * p->depth + 2;
  for (int t = 0; t < n; ++t) {
    int64_t off, rows, cols;
    const char* name;
    int layer;
    tensor_layout(p, t, &off, &rows, &cols, &name, &layer);
    float* base = (t == 0) ? p->wte : (t == n - 1 ? p->lm : p->blocks);
    float* dst = base + off;
    const int64_t numel = rows * cols;
    const bool out_proj = (layer >= 0) && ((t - 1) % 6 == 3 || (t - 1) % 6 == 5);
    const bool head = (t == n - 1);
    if (flags == NC_INIT_SPEC && (out_proj || head)) {
      NC_CUDA_TRY(cudaMemsetAsync(dst, 0, sizeof(float) * numel, p->stream));
      continue;
    }
    const double fan_in = (t == 0) ? 1.0 : (double)cols;
    const uint64_t key = splitmix64_host(seed ^ splitmix64_host((uint64_t)t + 1));
    NC_TRY(init_normal(dst, numel, key, (float)(1.0 / std::sqrt(fan_in)), p->stream));
  }
  return sync_bf16(p);
}

}  // namespace
}  // namespace nc

// ------------------------------------------------------------------ op status word
// One status word per device for the single-kernel entry points, which have
// no handle to carry one: a bounded wait that expires, a kernel that finds
// its shared memory misaligned or a token id out of range records its code
// here, and nc_op_sync returns it.  A file-scope __device__ variable, so no
// allocation is involved; its device address comes from
// cudaGetSymbolAddress (in host code the name only stands for the symbol).
namespace nc {
namespace {
__device__ int g_op_status;
constexpr int kMaxStatusDevices = 64;
std::mutex g_op_status_mu;
int* g_op_status_ptr[kMaxStatusDevices] = {};
}  // namespace

nc_status op_status_word(int** out) {
  int dev = 0;
  NC_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxStatusDevices) return fail(NC_ERR_UNSUPPORTED, "device index too large");
  std::lock_guard<std::mutex> lock(g_op_status_mu);
  if (!g_op_status_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_op_status);
    if (e != cudaSuccess || !ptr) return cuda_fail(e, "cudaGetSymbolAddress(op status word)");
    g_op_status_ptr[dev] = static_cast<int*>(ptr);
  }
  *out = g_op_status_ptr[dev];
  return NC_OK;
}
}  // namespace nc

// ==================================================================== C ABI
using namespace nc;

extern "C" {

const char* nc_last_error(void) { return g_last_error.c_str(); }

const char* nc_status_string(nc_status s) {
  switch (s) {
    case NC_OK: return "ok";
    case NC_ERR_INVALID_ARG: return "invalid argument";
    case NC_ERR_OOM: return "out of device memory";
    case NC_ERR_CUDA: return "CUDA error";
    case NC_ERR_TOKEN_RANGE: return "token id out of range";
    case NC_ERR_TIMEOUT: return "device wait timed out";
    case NC_ERR_UNSUPPORTED: return "unsupported";
  }
  return "unknown";
}

nc_status nc_gpt_init_config(const nc_model_config* cfg, nc_params** out) {
  if (!out || !cfg) return fail(NC_ERR_INVALID_ARG, "init: null argument");
  *out = nullptr;
  const int depth = cfg->depth, vocab = cfg->vocab, flags = cfg->flags;
  if (depth < 1 || depth > 32 || vocab < 8 || vocab > 32768 || vocab % 8 ||
      (flags != NC_INIT_SPEC && flags != NC_INIT_ALL_RANDOM))
    return fail(NC_ERR_INVALID_ARG, "init: depth in [1, 32], vocab in [8, 32768] (multiple of 8)");
  if (depth % 2)
    return fail(NC_ERR_UNSUPPORTED, "init: odd depth gives a head width other than 128");
  const int H = 64 * depth / 128;
  const int Hkv = cfg->n_kv_head > 0 ? cfg->n_kv_head : H;
  if (cfg->n_kv_head < 0 || Hkv > H || H % Hkv)
    return fail(NC_ERR_INVALID_ARG, "init: n_kv_head must divide the number of heads");
  nc_params* p = new nc_params();
  p->depth = depth;
  p->vocab = vocab;
  p->d = 64 * depth;
  p->hd = 128;
  p->H = H;
  p->Hkv = Hkv;
  p->dkv = 128 * Hkv;
  p->F = 4 * p->d;
  if (cfg->fp8 && p->d < 256) {
    delete p;
    return fail(NC_ERR_UNSUPPORTED, "init: fp8 mode needs d >= 256 (depth >= 4)");
  }
  p->fp8 = cfg->fp8 != 0;
  if (cfg->lm_chunk_tokens < 0) {
    delete p;
    return fail(NC_ERR_INVALID_ARG, "init: lm_chunk_tokens must be >= 0");
  }
  p->lm_chunk = cfg->lm_chunk_tokens > 0 ? cfg->lm_chunk_tokens : 32768;
  p->window.assign(depth, -1);
  if (cfg->window)
    for (int l = 0; l < depth; ++l) p->window[l] = cfg->window[l] < 0 ? -1 : cfg->window[l];
  p->prof = profiler_create();
  const int64_t d = p->d, V = vocab, be = block_elems(p), dkv = p->dkv;
  // Newton-Schulz stacks (see muon): squares, the dkv x d stack, the d x 4d
  // stack, and the workspace of the largest call (12 L d^2 covers each).
  const int64_t sq = (dkv == d ? 4ll : 2ll) * depth * d * d;
  const int64_t kvs = dkv == d ? 0 : 2ll * depth * dkv * d;
  const int64_t wide = 8ll * depth * d * d, ws = 12ll * depth * d * d;
  auto r = [](int64_t bytes) { return (bytes + 255) & ~int64_t(255); };
  const int64_t total = r(4 * V * d) * 2 + r(4 * be) * 2 + r(2 * be) + r(2 * V * d) +
                        r(4 * 6 * depth) + r(2 * sq) + r(2 * kvs) + r(2 * wide) + r(2 * ws) +
                        r(4);
  cudaError_t e = cudaMalloc(&p->pmem, (size_t)total);
  if (e != cudaSuccess) {
    cudaGetLastError();
    profiler_destroy(p->prof);
    delete p;
    return fail(NC_ERR_OOM, "parameter allocation failed");
  }
  Arena ar{static_cast<char*>(p->pmem), (size_t)total, 0};
  p->wte = ar.take<float>(V * d);
  p->lm = ar.take<float>(V * d);
  p->blocks = ar.take<float>(be);
  p->mom = ar.take<float>(be);
  p->blocks_b = ar.take<bf16>(be);
  p->lm_b = ar.take<bf16>(V * d);
  p->sumsq = ar.take<float>(6 * depth);
  p->xsq = ar.take<bf16>(sq);
  p->xkv = kvs ? ar.take<bf16>(kvs) : nullptr;
  p->xw = ar.take<bf16>(wide);
  p->nsws = ar.take<bf16>(ws);
  p->status = ar.take<int>(1);
  nc_status st = NC_OK;
  if (cudaMallocHost(&p->h_loss, sizeof(float)) != cudaSuccess ||
      cudaMallocHost(&p->h_status, sizeof(int)) != cudaSuccess)
    st = fail(NC_ERR_OOM, "pinned host allocation failed");
  if (st == NC_OK && cudaStreamCreateWithFlags(&p->wg, cudaStreamNonBlocking) != cudaSuccess)
    st = fail(NC_ERR_CUDA, "weight-gradient stream creation failed");
  for (int k = 0; k < 4 && st == NC_OK; ++k)
    if (cudaEventCreateWithFlags(&p->wg_fork[k], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&p->wg_done[k], cudaEventDisableTiming) != cudaSuccess)
      st = fail(NC_ERR_CUDA, "weight-gradient event creation failed");
  if (st == NC_OK && cudaMemsetAsync(p->mom, 0, sizeof(float) * be, p->stream) != cudaSuccess)
    st = fail(NC_ERR_CUDA, "momentum clear failed");
  if (st == NC_OK && cudaMemsetAsync(p->status, 0, sizeof(int), p->stream) != cudaSuccess)
    st = fail(NC_ERR_CUDA, "status clear failed");
  if (st == NC_OK) st = init_model(p, cfg->seed, flags);
  if (st == NC_OK && cudaStreamSynchronize(p->stream) != cudaSuccess)
    st = fail(NC_ERR_CUDA, "init synchronisation failed");
  if (st != NC_OK) {
    nc_params_free(p);
    return st;
  }
  *out = p;
  return NC_OK;
}

nc_status nc_gpt_init_ex(int depth, int vocab, uint64_t seed, int flags, nc_params** out) {
  nc_model_config cfg{};
  cfg.depth = depth;
  cfg.vocab = vocab;
  cfg.seed = seed;
  cfg.flags = flags;
  return nc_gpt_init_config(&cfg, out);
}

nc_status nc_gpt_init(int depth, int vocab, uint64_t seed, nc_params** out) {
  return nc_gpt_init_ex(depth, vocab, seed, NC_INIT_SPEC, out);
}

void nc_params_free(nc_params* p) {
  if (!p) return;
  if (p->stream) cudaStreamSynchronize(p->stream);
  else cudaDeviceSynchronize();
  drop_graph(p);
  if (p->wg) cudaStreamSynchronize(p->wg);
  for (int k = 0; k < 4; ++k) {
    if (p->wg_fork[k]) cudaEventDestroy(p->wg_fork[k]);
    if (p->wg_done[k]) cudaEventDestroy(p->wg_done[k]);
  }
  if (p->wg) cudaStreamDestroy(p->wg);
  if (p->act.mem) cudaFree(p->act.mem);
  if (p->rope) cudaFree(p->rope);
  if (p->adam) cudaFree(p->adam);
  if (p->pmem) cudaFree(p->pmem);
  if (p->h_loss) cudaFreeHost(p->h_loss);
  if (p->h_status) cudaFreeHost(p->h_status);
  profiler_destroy(p->prof);
  delete p;
}

nc_status nc_set_stream(nc_params* p, void* stream) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "set_stream: null handle");
  p->stream = static_cast<cudaStream_t>(stream);
  return NC_OK;
}

int nc_num_tensors(const nc_params* p) { return p ? 6 * p->depth + 2 : 0; }

nc_status nc_tensor_info(const nc_params* p, int idx, nc_tensor_desc* out) {
  if (!p || !out || idx < 0 || idx >= nc_num_tensors(p))
    return fail(NC_ERR_INVALID_ARG, "tensor_info: bad index");
  int64_t off, rows, cols;
  const char* name;
  int layer;
  tensor_layout(p, idx, &off, &rows, &cols, &name, &layer);
  std::memset(out, 0, sizeof(*out));
  if (layer >= 0) std::snprintf(out->name, sizeof(out->name), "h%d.%s", layer, name);
  else std::snprintf(out->name, sizeof(out->name), "%s", name);
  out->ndim = 2;
  out->shape[0] = rows;
  out->shape[1] = cols;
  out->dtype = NC_F32;
  const int n = nc_num_tensors(p);
  if (idx == 0) {
    out->data = p->wte;
    out->data_bf16 = nullptr;
  } else if (idx == n - 1) {
    out->data = p->lm;
    out->data_bf16 = p->lm_b;
  } else {
    out->data = p->blocks + off;
    out->data_bf16 = p->blocks_b + off;
  }
  return NC_OK;
}

nc_status nc_params_sync(nc_params* p) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "params_sync: null handle");
  return sync_bf16(p);
}

nc_status nc_tensor_write(nc_params* p, int idx, const float* src) {
  nc_tensor_desc t;
  NC_TRY(nc_tensor_info(p, idx, &t));
  if (!src) return fail(NC_ERR_INVALID_ARG, "tensor_write: null source");
  const int64_t n = t.shape[0] * t.shape[1];
  NC_CUDA_TRY(cudaMemcpyAsync(t.data, src, sizeof(float) * n, cudaMemcpyDefault, p->stream));
  if (t.data_bf16)
    NC_TRY(f32_to_bf16(static_cast<float*>(t.data), t.data_bf16, n, p->stream, nullptr));
  NC_CUDA_TRY(cudaStreamSynchronize(p->stream));
  return NC_OK;
}

nc_status nc_tensor_read(const nc_params* p, int idx, float* dst) {
  nc_tensor_desc t;
  NC_TRY(nc_tensor_info(p, idx, &t));
  if (!dst) return fail(NC_ERR_INVALID_ARG, "tensor_read: null destination");
  NC_CUDA_TRY(cudaMemcpyAsync(dst, t.data, sizeof(float) * t.shape[0] * t.shape[1],
                              cudaMemcpyDefault, p->stream));
  NC_CUDA_TRY(cudaStreamSynchronize(p->stream));
  return NC_OK;
}

nc_status nc_momentum_read(const nc_params* p, int idx, float* dst) {
  if (!p || !dst || idx < 1 || idx > 6 * p->depth)
    return fail(NC_ERR_INVALID_ARG, "momentum_read: bad index");
  int64_t off, rows, cols;
  const char* name;
  int layer;
  tensor_layout(p, idx, &off, &rows, &cols, &name, &layer);
  NC_CUDA_TRY(cudaMemcpyAsync(dst, p->mom + off, sizeof(float) * rows * cols, cudaMemcpyDefault,
                              p->stream));
  NC_CUDA_TRY(cudaStreamSynchronize(p->stream));
  return NC_OK;
}

nc_status nc_grads_create(const nc_params* p, nc_grads** out) {
  if (!p || !out) return fail(NC_ERR_INVALID_ARG, "grads_create: null argument");
  nc_grads* g = new nc_grads();
  g->p = p;
  const int64_t vd = (int64_t)p->vocab * p->d, be = block_elems(p);
  cudaError_t e = cudaMalloc(&g->mem, sizeof(float) * (2 * vd + be));
  if (e != cudaSuccess) {
    cudaGetLastError();
    delete g;
    return fail(NC_ERR_OOM, "gradient allocation failed");
  }
  g->wte = static_cast<float*>(g->mem);
  g->lm = g->wte + vd;
  g->blocks = g->lm + vd;
  *out = g;
  return NC_OK;
}

void nc_grads_free(nc_grads* g) {
  if (!g) return;
  cudaDeviceSynchronize();
  if (g->p && g->p->graph_g == g) drop_graph(const_cast<nc_params*>(g->p));
  if (g->mem) cudaFree(g->mem);
  delete g;
}

nc_status nc_grad_info(const nc_grads* g, int idx, nc_tensor_desc* out) {
  if (!g) return fail(NC_ERR_INVALID_ARG, "grad_info: null handle");
  NC_TRY(nc_tensor_info(g->p, idx, out));
  int64_t off, rows, cols;
  const char* name;
  int layer;
  tensor_layout(g->p, idx, &off, &rows, &cols, &name, &layer);
  const int n = nc_num_tensors(g->p);
  out->data = idx == 0 ? g->wte : (idx == n - 1 ? g->lm : g->blocks + off);
  out->data_bf16 = nullptr;
  return NC_OK;
}

nc_status nc_grad_read(const nc_grads* g, int idx, float* dst) {
  nc_tensor_desc t;
  NC_TRY(nc_grad_info(g, idx, &t));
  if (!dst) return fail(NC_ERR_INVALID_ARG, "grad_read: null destination");
  NC_CUDA_TRY(cudaMemcpyAsync(dst, t.data, sizeof(float) * t.shape[0] * t.shape[1],
                              cudaMemcpyDefault, g->p->stream));
  NC_CUDA_TRY(cudaStreamSynchronize(g->p->stream));
  return NC_OK;
}

nc_status nc_grad_write(nc_grads* g, int idx, const float* src) {
  nc_tensor_desc t;
  NC_TRY(nc_grad_info(g, idx, &t));
  if (!src) return fail(NC_ERR_INVALID_ARG, "grad_write: null source");
  NC_CUDA_TRY(cudaMemcpyAsync(t.data, src, sizeof(float) * t.shape[0] * t.shape[1],
                              cudaMemcpyDefault, g->p->stream));
  NC_CUDA_TRY(cudaStreamSynchronize(g->p->stream));
  return NC_OK;
}

nc_status nc_gpt_fwd_bwd_async(nc_params* p, const int32_t* tokens, const int32_t* targets, int B,
                               int T, float* loss_dev, nc_grads* g) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "fwd_bwd: null handle");
  return fwd_bwd(p, tokens, targets, B, T, loss_dev, g);
}

nc_status nc_gpt_fwd_bwd(nc_params* p, const int32_t* tokens, const int32_t* targets, int B,
                         int T, float* loss_host, nc_grads* g) {
  if (!p || !loss_host) return fail(NC_ERR_INVALID_ARG, "fwd_bwd: null argument");
  NC_TRY(fwd_bwd(p, tokens, targets, B, T, nullptr, g));
  NC_TRY(sync_and_check(p, p->act.loss));
  *loss_host = *p->h_loss;
  return NC_OK;
}

nc_status nc_muon_step(nc_params* p, const nc_grads* g, float lr, float momentum) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "muon: null handle");
  return muon(p, g, lr, momentum);
}

nc_status nc_step_capture(nc_params* p, const int32_t* tokens, const int32_t* targets, int B, int T,
                          float* loss_dev, nc_grads* g, float lr, float momentum) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "step_capture: null handle");
  if (p->poisoned) return fail(NC_ERR_TIMEOUT, "handle poisoned by an earlier device timeout");
  if (!p->stream)
    return fail(NC_ERR_INVALID_ARG, "step_capture: set a non-default stream first (nc_set_stream)");
  if (!tokens || !targets || !loss_dev || !g || g->p != p || B < 1 || T < 1 ||
      (int64_t)B * T > (1 << 24))
    return fail(NC_ERR_INVALID_ARG, "step_capture: bad arguments");
  if (!is_device_ptr(tokens) || !is_device_ptr(targets) || !is_device_ptr(loss_dev))
    return fail(NC_ERR_INVALID_ARG, "step_capture: tokens, targets and loss must be device memory");
  // Everything that allocates happens before the capture.
  NC_TRY(ensure_acts(p, B, T));
  NC_TRY(ensure_rope(p, T));
  drop_graph(p);
  const bool prof_on = profiler_enabled(p->prof);
  profiler_enable(p->prof, false);
  const int64_t launches0 = profiler_launches(p->prof);
  cudaError_t e = cudaStreamBeginCapture(p->stream, cudaStreamCaptureModeRelaxed);
  if (e != cudaSuccess) {
    profiler_enable(p->prof, prof_on);
    return cuda_fail(e, "step_capture: begin capture");
  }
  nc_status st = fwd_bwd(p, tokens, targets, B, T, loss_dev, g, true);
  if (st == NC_OK) st = muon(p, g, lr, momentum);
  cudaGraph_t graph = nullptr;
  e = cudaStreamEndCapture(p->stream, &graph);  // always ends the capture
  profiler_enable(p->prof, prof_on);
  const int64_t n = profiler_launches(p->prof) - launches0;
  profiler_add_launches(p->prof, -n);  // recorded, not run
  if (st != NC_OK || e != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    return st != NC_OK ? st : cuda_fail(e, "step_capture: end capture");
  }
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, graph, 0);
  if (e != cudaSuccess) {
    cudaGraphDestroy(graph);
    return cuda_fail(e, "step_capture: instantiate");
  }
  p->graph = graph;
  p->graph_exec = exec;
  p->graph_launches = n;
  p->graph_g = g;
  return NC_OK;
}

nc_status nc_step_replay(nc_params* p) {
  if (!p || !p->graph_exec) return fail(NC_ERR_INVALID_ARG, "step_replay: no captured step");
  if (p->poisoned) return fail(NC_ERR_TIMEOUT, "handle poisoned by an earlier device timeout");
  if (!p->stream) return fail(NC_ERR_INVALID_ARG, "step_replay: the handle's stream was reset");
  NC_CUDA_TRY(cudaGraphLaunch(p->graph_exec, p->stream));
  profiler_add_launches(p->prof, p->graph_launches);
  return NC_OK;
}

nc_status nc_adamw_step(nc_params* p, const nc_grads* g, float lr_embed, float lr_head, float beta1,
                        float beta2, float eps, float weight_decay) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "adamw: null handle");
  if (p->poisoned) return fail(NC_ERR_TIMEOUT, "handle poisoned by an earlier device timeout");
  if (!g || g->p != p) return fail(NC_ERR_INVALID_ARG, "adamw: gradients of another model");
  if (!(lr_embed >= 0.f) || !(lr_head >= 0.f) || !(beta1 >= 0.f && beta1 < 1.f) ||
      !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f) || !(weight_decay >= 0.f))
    return fail(NC_ERR_INVALID_ARG, "adamw: lr, eps, weight_decay >= 0 and betas in [0, 1)");
  const int64_t n = (int64_t)p->vocab * p->d;  // wte and lm_head are both [V, d]
  if (!p->adam) {
    NC_CUDA_TRY(cudaMalloc(&p->adam, sizeof(float) * 4 * n));
    NC_CUDA_TRY(cudaMemsetAsync(p->adam, 0, sizeof(float) * 4 * n, p->stream));
  }
  const int t = ++p->adam_t;
  NC_TRY(adamw(p->wte, nullptr, p->adam, p->adam + n, g->wte, n, lr_embed, beta1, beta2, eps,
               weight_decay, t, p->stream, p->prof));
  NC_TRY(adamw(p->lm, p->lm_b, p->adam + 2 * n, p->adam + 3 * n, g->lm, n, lr_head, beta1, beta2,
               eps, weight_decay, t, p->stream, p->prof));
  return NC_OK;
}

nc_status nc_sync(nc_params* p) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "sync: null handle");
  return sync_and_check(p, nullptr);
}

int* nc_debug_status_word(nc_params* p) { return p ? p->status : nullptr; }

nc_status nc_profile_enable(nc_params* p, int on) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "profile: null handle");
  profiler_enable(p->prof, on != 0);
  return NC_OK;
}

nc_status nc_profile_read(nc_params* p, nc_kernel_stat* out, int max, int* n) {
  if (!p || !out || max < 0) return fail(NC_ERR_INVALID_ARG, "profile: bad arguments");
  return profiler_read(p->prof, out, max, n);
}

int64_t nc_launch_count(const nc_params* p) { return p ? profiler_launches(p->prof) : 0; }

// ------------------------------------------------------------------ ops
nc_status nc_op_gemm(const nc_gemm_desc* desc, void* stream) {
  if (!desc) return fail(NC_ERR_INVALID_ARG, "gemm: null descriptor");
  GemmLaunch g{};
  g.d = *desc;
  NC_TRY(op_status_word(&g.status));
  if (g.d.split_k < 0) return fail(NC_ERR_INVALID_ARG, "gemm: split_k < 0");
  if (g.d.split_k == 0) g.d.split_k = 1;
  return gemm_launch(g, static_cast<cudaStream_t>(stream), nullptr);
}

nc_status nc_op_rmsnorm(const float* x, int64_t rows, int cols, void* y_bf16, float* rstd,
                        void* stream) {
  if (!x || !y_bf16 || rows < 0 || cols < 4) return fail(NC_ERR_INVALID_ARG, "rmsnorm: bad arguments");
  if (rows == 0) return NC_OK;
  return rmsnorm_fwd(x, rows, cols, y_bf16, rstd, static_cast<cudaStream_t>(stream), nullptr);
}

nc_status nc_op_embed_gather(const int32_t* tokens, int64_t n, const float* E, int vocab, int d,
                             float* x, void* stream) {
  if (n < 0 || vocab < 1 || d < 4 || d % 4 || (n > 0 && (!tokens || !E || !x)))
    return fail(NC_ERR_INVALID_ARG, "embed_gather: bad arguments (d a positive multiple of 4)");
  if ((reinterpret_cast<uintptr_t>(E) | reinterpret_cast<uintptr_t>(x)) & 15)
    return fail(NC_ERR_INVALID_ARG, "embed_gather: E and x must be 16-byte aligned");
  if (n == 0) return NC_OK;
  int* st = nullptr;
  NC_TRY(op_status_word(&st));
  return embed_gather(tokens, n, E, vocab, d, x, st, static_cast<cudaStream_t>(stream), nullptr);
}

nc_status nc_op_fp8_quantize(const void* x, int x_bf16, int64_t rows, int cols, int64_t ldx, int transpose,
                             void* q, int64_t ldq, float* scale, void* scratch, void* stream) {
  if (!x || !q || !scale || !scratch || rows < 1 || cols < 8 || cols % 8 || ldx < cols || ldx % 8 ||
      (transpose && rows % 8) || ldq % 16 || ldq < (transpose ? rows : (int64_t)cols))
    return fail(NC_ERR_INVALID_ARG, "fp8_quantize: bad arguments (cols and ldx multiples of 8, rows too "
                                    "when transposing, ldq a multiple of 16)");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(q)) & 15)
    return fail(NC_ERR_INVALID_ARG, "fp8_quantize: x and q must be 16-byte aligned");
  return fp8_quantize(x, x_bf16 != 0, rows, cols, ldx, transpose != 0, static_cast<uint8_t*>(q), ldq, scale,
                      static_cast<unsigned*>(scratch), static_cast<cudaStream_t>(stream), nullptr);
}

nc_status nc_op_fp8_quantize2(const void* x_bf16, int64_t rows, int cols, int64_t ldx, void* q, void* qT,
                              float* scale, void* scratch, void* stream) {
  if (!x_bf16 || (!q && !qT) || !scale || !scratch || rows < 8 || rows % 8 || cols < 8 || cols % 8 ||
      ldx < cols || ldx % 8)
    return fail(NC_ERR_INVALID_ARG, "fp8_quantize2: bad arguments (rows, cols and ldx multiples of 8)");
  if ((reinterpret_cast<uintptr_t>(x_bf16) | reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(qT)) & 15)
    return fail(NC_ERR_INVALID_ARG, "fp8_quantize2: x, q and qT must be 16-byte aligned");
  return fp8_quantize2(x_bf16, rows, cols, ldx, static_cast<uint8_t*>(q), static_cast<uint8_t*>(qT), scale,
                       nullptr, static_cast<unsigned*>(scratch), false, static_cast<cudaStream_t>(stream), nullptr);
}

nc_status nc_op_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return fail(NC_ERR_INVALID_ARG, "exp2_poly: bad arguments");
  if (n == 0) return NC_OK;
  return exp2_poly(x, y, n, static_cast<cudaStream_t>(stream));
}

nc_status nc_op_sync(void* stream) {
  int* word = nullptr;
  NC_TRY(op_status_word(&word));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h = 0;
  NC_CUDA_TRY(cudaMemcpyAsync(&h, word, sizeof(int), cudaMemcpyDeviceToHost, s));
  NC_CUDA_TRY(cudaStreamSynchronize(s));
  if (h == kDevOk) return NC_OK;
  NC_CUDA_TRY(cudaMemsetAsync(word, 0, sizeof(int), s));
  NC_CUDA_TRY(cudaStreamSynchronize(s));
  if (h == kDevTimeout)
    return fail(NC_ERR_TIMEOUT, "an op's bounded device wait expired (or its shared memory was "
                                "misaligned); its outputs are incomplete");
  if (h == kDevTokenRange) return fail(NC_ERR_TOKEN_RANGE, "an op read a token id out of [0, vocab)");
  return fail(NC_ERR_CUDA, "unknown op status");
}

int* nc_debug_op_status_word(void) {
  int* word = nullptr;
  return op_status_word(&word) == NC_OK ? word : nullptr;
}

nc_status nc_op_attention_fwd(const void* q, const void* k, const void* v, int64_t ld, void* o,
                              int64_t ldo, float* lse, int B, int T, int H, void* stream) {
  int* st = nullptr;
  NC_TRY(op_status_word(&st));
  return attention_fwd(q, k, v, ld, o, ldo, lse, B, T, H, st, static_cast<cudaStream_t>(stream),
                       nullptr);
}

nc_status nc_op_attention_bwd(const void* q, const void* k, const void* v, int64_t ld,
                              const void* o, const void* dout, int64_t ldo, const float* lse,
                              float* dq, void* dk, void* dv, int64_t ldg, float* delta_scratch,
                              int B, int T, int H, void* stream) {
  int* st = nullptr;
  NC_TRY(op_status_word(&st));
  return attention_bwd(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta_scratch, B, T, H,
                       st, static_cast<cudaStream_t>(stream), nullptr);
}

nc_status nc_op_attention_fwd_ex(const void* q, int64_t ldq, const void* k, const void* v,
                                 int64_t ldkv, void* o, int64_t ldo, float* lse, int B, int T, int H,
                                 int Hkv, int window, void* stream) {
  int* st = nullptr;
  NC_TRY(op_status_word(&st));
  return attention_fwd_ex(q, ldq, k, v, ldkv, o, ldo, lse, B, T, H, Hkv, window, st,
                          static_cast<cudaStream_t>(stream), nullptr);
}

nc_status nc_op_attention_bwd_ex(const void* q, int64_t ldq, const void* k, const void* v,
                                 int64_t ldkv, const void* o, const void* dout, int64_t ldo,
                                 const float* lse, float* dq, void* dk, void* dv, int64_t ldg,
                                 float* delta_scratch, int B, int T, int H, int Hkv, int window,
                                 void* stream) {
  int* st = nullptr;
  NC_TRY(op_status_word(&st));
  return attention_bwd_ex(q, ldq, k, v, ldkv, o, dout, ldo, lse, dq, dk, dv, ldg, delta_scratch, B,
                          T, H, Hkv, window, st, static_cast<cudaStream_t>(stream), nullptr);
}

size_t nc_newton_schulz_scratch_bytes(int count, int rows, int cols) {
  if (count < 1 || rows < 1 || cols < 1) return 0;
  const int64_t m = std::min(rows, cols), n = std::max(rows, cols);
  // X (normalised, wide) + A + B + second X, then the fp32 norms.
  return (size_t)(2 * (count * m * n) + 2 * (count * m * m)) * 2 + (size_t)count * 4 + 256;
}

nc_status nc_op_newton_schulz(const void* x_bf16, void* out_bf16, int count, int rows, int cols,
                              int steps, void* scratch, void* stream) {
  if (!x_bf16 || !out_bf16 || !scratch || count < 1 || rows < 1 || cols < 1 || steps < 0)
    return fail(NC_ERR_INVALID_ARG, "newton_schulz: bad arguments");
  if (((int64_t)rows * cols) % 8 || std::min(rows, cols) % 8)
    return fail(NC_ERR_INVALID_ARG, "newton_schulz: dims must be multiples of 8");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int m = std::min(rows, cols), n = std::max(rows, cols);
  const bool tall = rows > cols;
  const int64_t mn = (int64_t)m * n;
  bf16* X = static_cast<bf16*>(scratch);
  bf16* ws = X + count * mn;  // A, B, second X
  float* norms = reinterpret_cast<float*>(ws + count * mn + 2 * (int64_t)count * m * m);
  NC_CUDA_TRY(cudaMemsetAsync(norms, 0, sizeof(float) * count, s));
  NC_TRY(sumsq_bf16(x_bf16, mn, count, norms, s, nullptr));
  NC_TRY(scale_bf16(x_bf16, rows, cols, tall ? 1 : 0, norms, 1e-7f, X, count, s, nullptr));
  int* st = nullptr;
  NC_TRY(op_status_word(&st));
  NC_TRY(newton_schulz_wide(X, count, m, n, steps, ws, st, s, nullptr));
  // Back to the caller's orientation (no scaling).
  NC_TRY(scale_bf16(X, m, n, tall ? 1 : 0, nullptr, 0.f, out_bf16, count, s, nullptr));
  return NC_OK;
}

}  // extern "C"
