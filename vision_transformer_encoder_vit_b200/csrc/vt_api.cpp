// C ABI of libvt (declared in include/vt.h): handle, configuration checks, weight
// table, workspace plan, launch sequences, error reporting and launch profiling.
// Host code only; every step of the computation runs in the kernels of gemm.cu,
// attention.cu and elementwise.cu.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/vt.h"
#include "internal.h"

using namespace vt;

namespace {

thread_local std::string g_last_error;

vt_status fail(vt_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

vt_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int round8(int x) { return (x + 7) & ~7; }

// ---------------------------------------------------------------- profiling

enum {
  CLS_GEMM = 0,
  CLS_ATTN = 1,
  CLS_LN = 2,
  CLS_UNFOLD = 3,
  CLS_REORDER = 4,
  CLS_PREP = 5,
  CLS_ATTN_BWD = 6,
  CLS_BWD_MISC = 7,
  CLS_COUNT = 8
};

struct ProfRec {
  int cls;
  cudaEvent_t a, b;
  double flops, bytes;
  int kernels;  // kernels the bracketed call launched
};

struct DoneRec {
  int cls;
  double ms, flops, bytes;
};

struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<DoneRec> done;  // resolved launches of the last profiled interval
  std::vector<cudaEvent_t> pool;
  double ms[CLS_COUNT] = {0}, flops[CLS_COUNT] = {0}, bytes[CLS_COUNT] = {0};
  int64_t n[CLS_COUNT] = {0};
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e;
    cudaEventCreate(&e);
    return e;
  }
};
Profiler g_prof;

// Launch trace: with VT_LOG set to anything but empty or "0" when the library loads,
// every launch is written to stderr as it is issued (kernel class, algorithmic FLOPs
// and bytes, stream).  Host side only, so it also traces launches recorded into a CUDA
// graph; off, it costs one branch per launch.
const char* const kClassNames[CLS_COUNT] = {"gemm",           "attention",          "layernorm",
                                            "patch_unfold",   "reorder",            "attention_prep",
                                            "attention_backward", "backward_misc"};
const bool g_log = [] {
  const char* v = std::getenv("VT_LOG");
  return v != nullptr && v[0] != '\0' && !(v[0] == '0' && v[1] == '\0');
}();

// Brackets one launch with events when profiling is on; traces it when VT_LOG is set.
struct ProfScope {
  int cls;
  double flops, bytes;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  int kernels = 1;
  ProfScope(int c, double f, double b, cudaStream_t s) : cls(c), flops(f), bytes(b), st(s) {
    if (g_log)
      std::fprintf(stderr, "vt: launch %s flops=%.6g bytes=%.6g stream=%p\n", kClassNames[c], f, b,
                   static_cast<void*>(s));
    if (g_prof.on) {
      std::lock_guard<std::mutex> l(g_prof.mu);
      a = g_prof.get();
      cudaEventRecord(a, st);
    }
  }
  ~ProfScope() {
    if (a) {
      std::lock_guard<std::mutex> l(g_prof.mu);
      cudaEvent_t b = g_prof.get();
      cudaEventRecord(b, st);
      g_prof.recs.push_back({cls, a, b, flops, bytes, kernels});
    }
  }
};

// ------------------------------------------------------------ kernel calls

vt_status run_gemm(GemmParams p, cudaStream_t st) {
  ProfScope ps(CLS_GEMM, 2.0 * p.M * static_cast<double>(p.N) * p.K, 0, st);
  cudaError_t e = launch_gemm(p, st, 0, &ps.kernels);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return VT_OK;
}

// The same product with a split-K tail allowed, on `scratch` (gemm_split_bytes()).
GemmParams split_k(GemmParams p, char* scratch) {
  p.sk_part = reinterpret_cast<float*>(scratch);
  return p;
}

GemmParams gemm_params(const void* A, int lda, const void* W, int ldw, const void* bias, const void* resid,
                       int ldr, void* out, int ldo, int M, int N, int K, int act) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.A = A;
  p.lda = lda;
  p.W = W;
  p.ldw = ldw;
  p.bias = bias;
  p.resid = resid;
  p.ldr = ldr;
  p.out = out;
  p.ldo = ldo;
  p.M = M;
  p.N = N;
  p.K = K;
  p.act = act;
  return p;
}

vt_status run_layernorm(const void* x, const void* g, const void* b, void* y, int rows, int cols, float eps,
                        cudaStream_t st) {
  ProfScope ps(CLS_LN, 0, 4.0 * rows * static_cast<double>(cols), st);
  cudaError_t e = launch_layernorm(x, g, b, y, rows, cols, eps, st);
  if (e != cudaSuccess) return cuda_fail(e, "layernorm launch");
  return VT_OK;
}

}  // namespace

vt_status vt::run_attention(const AttnParams& p, cudaStream_t st) {
  double n2 = static_cast<double>(p.B) * p.N * p.N, n1 = static_cast<double>(p.B) * p.N;
  if (p.varlen) {  // per-image token counts of a packed batch
    n2 = n1 = 0;
    for (int b = 0; b < p.vl.count; ++b) {
      const double n = p.vl.tok_off[b + 1] - p.vl.tok_off[b];
      n2 += n * n;
      n1 += n;
    }
  }
  ProfScope ps(CLS_ATTN, 4.0 * p.H * n2 * p.D, 8.0 * p.H * n1 * p.D, st);
  cudaError_t e = launch_attention(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return VT_OK;
}

vt_status vt::run_attention_prep(const void* q, const void* k, const void* v, void* qr, void* kr, void* vt_, int B,
                                 int H, int N, int D, int ld_vt, const int32_t* pos, const int sections[3],
                                 float theta, cudaStream_t st) {
  ProfScope ps(CLS_PREP, 0, 12.0 * B * H * static_cast<double>(N) * D, st);
  cudaError_t e = launch_attention_prep(q, k, v, qr, kr, vt_, B, H, N, D, ld_vt, pos, sections, theta, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention preparation launch");
  return VT_OK;
}

vt_status vt::check_attention_dims(int B, int H, int N, int D, float scale) {
  if (B <= 0 || H <= 0 || N <= 0) return fail(VT_ERR_INVALID_ARG, "B, H, N must be positive");
  if (!(scale > 0.f)) return fail(VT_ERR_INVALID_ARG, "scale must be positive");
  if (D != 32 && D != 64 && D != 80 && D != 96) return fail(VT_ERR_UNSUPPORTED, "head_dim %d has no kernel", D);
  if (static_cast<long long>(B) * H * N > (1ll << 31) - 256) return fail(VT_ERR_SHAPE, "too many rows");
  return VT_OK;
}

void vt::set_error_message(const char* msg) { g_last_error = msg ? msg : ""; }

// ------------------------------------------------------------------ handle

struct vt_handle {
  vt_config cfg;
  bool loaded = false;
  struct Layer {
    const void *ln1_w, *ln1_b, *qkv_w, *qkv_b, *o_w, *o_b, *ln2_w, *ln2_b, *fc1_w, *fc1_b, *fc2_w, *fc2_b;
  };
  const void *pe_w = nullptr, *pe_b = nullptr;
  std::vector<Layer> layers;
  const void *pa1_w, *pa1_b, *pa2_w, *pa2_b, *pb1_w, *pb1_b, *pb2_w, *pb2_b;
  void* qkv_pack = nullptr;  // owned: fused [3d, d] weights + [3d] biases per layer
  float2* rope_tab = nullptr;  // owned: [3][kRopeMaxPos][kRopePairs]
  // Backward (vt_enable_backward): transposed weights, so every input-gradient product
  // is a K-major GEMM.  qkv_t [d, 3d], o_t [d, d], fc1_t [d, m], fc2_t [m, d], pe_t [K0, d].
  struct LayerT {
    void *qkv_t, *o_t, *fc1_t, *fc2_t;
  };
  std::vector<LayerT> layers_t;
  void* pe_t = nullptr;
  void* bwd_pack = nullptr;  // owned: all of the above
};

namespace {

bool qkv_layout_supported(const vt_config& c) {
  if (c.head_dim == 80 && c.rope_sections[0] == 16 && c.rope_sections[1] == 32 && c.rope_sections[2] == 32) return true;
  if (c.head_dim == 32 && c.rope_sections[0] == 8 && c.rope_sections[1] == 12 && c.rope_sections[2] == 12) return true;
  return false;
}

struct Plan {
  int N, M, Mm, ld_vt;
  size_t x, sk, xn, q, k, vt, o, hmid, unfold, y1, y2, z1, total;
};

// Workspace layout for M packed tokens whose transposed v blocks take vt_elems elements.
Plan make_plan_core(const vt_config& c, int M_, size_t vt_elems) {
  Plan p;
  p.N = 0;
  p.ld_vt = 0;
  p.M = M_;
  p.Mm = M_ / 4;
  const size_t d = c.hidden, M = static_cast<size_t>(M_);
  const size_t K0 = 3ull * c.temporal_patch * c.patch * c.patch;
  size_t off = 0;
  p.x = off;
  off += align256(M * d * 2);
  p.sk = off;  // split-K scratch of the linear layers (fixed size)
  off += align256(gemm_split_bytes());
  const size_t base = off;
  // tower phase
  size_t o2 = base;
  p.xn = o2;
  o2 += align256(M * d * 2);
  p.q = o2;
  o2 += align256(M * d * 2);
  p.k = o2;
  o2 += align256(M * d * 2);
  p.vt = o2;
  o2 += align256(vt_elems * 2);
  p.o = o2;
  o2 += align256(M * d * 2);
  p.hmid = o2;
  o2 += align256(M * std::max<size_t>(c.mlp, K0) * 2);
  p.unfold = p.hmid;  // only live before the first layer
  // projector phase (reuses the tower-phase space)
  size_t o3 = base;
  p.y1 = o3;
  o3 += align256(M * static_cast<size_t>(c.proj_hidden) * 2);
  p.y2 = o3;
  o3 += align256(M * static_cast<size_t>(c.proj_hidden) * 2);
  p.z1 = o3;
  o3 += align256(static_cast<size_t>(p.Mm) * c.proj_hidden * 2);
  p.total = std::max(o2, o3);
  return p;
}

Plan make_plan(const vt_config& c, int B, int t, int h, int w) {
  const int N = t * h * w;
  const int ld = round8(N);
  Plan p = make_plan_core(c, B * N, static_cast<size_t>(B) * c.heads * c.head_dim * ld);
  p.N = N;
  p.ld_vt = ld;
  return p;
}

vt_status check_grid(const vt_handle* h, int B, const int32_t* g, int* t, int* gh, int* gw) {
  if (!g) return fail(VT_ERR_INVALID_ARG, "grid_thw is NULL");
  if (B <= 0) return fail(VT_ERR_INVALID_ARG, "batch must be positive (got %d)", B);
  *t = g[0];
  *gh = g[1];
  *gw = g[2];
  if (*t <= 0 || *gh <= 0 || *gw <= 0) return fail(VT_ERR_INVALID_ARG, "grid_thw must be positive");
  if (*t > kRopeMaxPos) return fail(VT_ERR_SHAPE, "t = %d above %d temporal patches", *t, kRopeMaxPos);
  if ((*gh % h->cfg.merge) || (*gw % h->cfg.merge))
    return fail(VT_ERR_SHAPE, "grid %dx%d is not a multiple of the %dx%d merge", *gh, *gw, h->cfg.merge, h->cfg.merge);
  if (*gh > kRopeMaxPos || *gw > kRopeMaxPos)
    return fail(VT_ERR_SHAPE, "grid side above %d patches", kRopeMaxPos);
  const long long M = static_cast<long long>(B) * (*t) * (*gh) * (*gw);
  if (M > (1ll << 30)) return fail(VT_ERR_SHAPE, "too many tokens in one call (%lld)", M);
  return VT_OK;
}

// Entry points whose pixels are still images [B, 3, H, W] take grids with t = 1 only.
vt_status check_still(int t, const char* entry) {
  if (t != 1)
    return fail(VT_ERR_SHAPE, "%s takes still images (t = 1), got t = %d; clips go through vt_forward_video", entry, t);
  return VT_OK;
}

// The patch-embedding product: patch vectors U [M, K0] -> tokens x [M, hidden].
vt_status run_patch_embed(vt_handle* h, const void* U, void* x, char* ws, const Plan& pl, cudaStream_t st) {
  const vt_config& c = h->cfg;
  const int K0 = 3 * c.temporal_patch * c.patch * c.patch;
  return run_gemm(
      split_k(gemm_params(U, K0, h->pe_w, K0, h->pe_b, nullptr, 0, x, c.hidden, pl.M, c.hidden, K0, ACT_NONE), ws + pl.sk),
      st);
}

// One pre-LN layer over the M tokens at x_in (written to x, which may equal x_in).  With
// vl non-null the tokens are a packed batch of images of different grids.
vt_status run_layer(vt_handle* h, int i, const void* x_in, void* x, int B, int gt, int gh, int gw, int order,
                    char* ws, const Plan& pl, cudaStream_t st, const VarlenTable* vl = nullptr) {
  const vt_config& c = h->cfg;
  const vt_handle::Layer& L = h->layers[i];
  const int d = c.hidden, M = pl.M;
  void* xn = ws + pl.xn;
  vt_status s = run_layernorm(x_in, L.ln1_w, L.ln1_b, xn, M, d, c.ln_eps, st);
  if (s) return s;
  {
    GemmParams p = gemm_params(xn, d, L.qkv_w, d, L.qkv_b, nullptr, 0, nullptr, 0, M, 3 * d, d, ACT_NONE);
    p.q = ws + pl.q;
    p.k = ws + pl.k;
    p.vt = ws + pl.vt;
    p.heads = c.heads;
    p.head_dim = c.head_dim;
    p.ntok = pl.N;
    p.ld_vt = pl.ld_vt;
    p.gt = gt;
    p.gh = gh;
    p.gw = gw;
    p.order = order;
    p.rope = c.use_rope;
    p.sections[0] = c.rope_sections[0];
    p.sections[1] = c.rope_sections[1];
    p.sections[2] = c.rope_sections[2];
    p.rope_tab = h->rope_tab;
    if (vl) {
      p.varlen = 1;
      p.vl = *vl;
    }
    ProfScope ps(CLS_GEMM, 2.0 * M * 3.0 * d * d, 0, st);
    cudaError_t e = launch_gemm(p, st, 1);
    if (e != cudaSuccess) return cuda_fail(e, "qkv gemm launch");
  }
  {
    AttnParams a{};
    a.q = ws + pl.q;
    a.k = ws + pl.k;
    a.vt = ws + pl.vt;
    a.o = ws + pl.o;
    a.B = B;
    a.H = c.heads;
    a.N = pl.N;
    a.D = c.head_dim;
    a.ld_vt = pl.ld_vt;
    a.scale = 1.0f / std::sqrt(static_cast<float>(c.head_dim));
    if (vl) {
      // one launch for the whole packed batch: per-image token counts come from the
      // table; v^T blocks share the stride ld_vt[0] (>= every image's tokens)
      a.varlen = 1;
      a.vl = *vl;
      a.B = vl->count;
      int nmax = 0;
      for (int b = 0; b < vl->count; ++b) nmax = std::max(nmax, vl->tok_off[b + 1] - vl->tok_off[b]);
      a.N = nmax;
      a.ld_vt = vl->ld_vt[0];
    }
    if ((s = run_attention(a, st))) return s;
  }
  if ((s = run_gemm(split_k(gemm_params(ws + pl.o, d, L.o_w, d, L.o_b, x_in, d, x, d, M, d, d, ACT_NONE), ws + pl.sk),
                    st)))
    return s;
  if ((s = run_layernorm(x, L.ln2_w, L.ln2_b, xn, M, d, c.ln_eps, st))) return s;
  const int act = c.gelu_tanh ? ACT_GELU_TANH : ACT_GELU_ERF;
  if ((s = run_gemm(gemm_params(xn, d, L.fc1_w, d, L.fc1_b, nullptr, 0, ws + pl.hmid, c.mlp, M, c.mlp, d, act), st)))
    return s;
  return run_gemm(
      split_k(gemm_params(ws + pl.hmid, c.mlp, L.fc2_w, c.mlp, L.fc2_b, x, d, x, d, M, d, c.mlp, ACT_NONE), ws + pl.sk),
      st);
}

// Projector on block-ordered tokens x [M, d] -> out [M/4, proj_out].
vt_status run_projector(vt_handle* h, const void* x, void* out, char* ws, const Plan& pl, cudaStream_t st) {
  const vt_config& c = h->cfg;
  const int d = c.hidden, P = c.proj_hidden, M = pl.M, Mm = pl.Mm;
  const int act = c.proj_gelu_tanh ? ACT_GELU_TANH : ACT_GELU_ERF;
  auto gemm = [&](const void* A, int lda, const void* W, const void* b, void* o, int ldo, int rows, int n, int k,
                  int a) { return run_gemm(split_k(gemm_params(A, lda, W, lda, b, nullptr, 0, o, ldo, rows, n, k, a),
                                                   ws + pl.sk),
                                           st); };
  vt_status s;
  if ((s = gemm(x, d, h->pa1_w, h->pa1_b, ws + pl.y1, P, M, P, d, act))) return s;
  if ((s = gemm(ws + pl.y1, P, h->pa2_w, h->pa2_b, ws + pl.y2, P, M, P, P, ACT_NONE))) return s;
  // Four consecutive block-ordered rows of y2 are one merged token: a [M/4, 4P] view.
  if ((s = gemm(ws + pl.y2, 4 * P, h->pb1_w, h->pb1_b, ws + pl.z1, P, Mm, P, 4 * P, act))) return s;
  return gemm(ws + pl.z1, P, h->pb2_w, h->pb2_b, out, c.proj_out, Mm, c.proj_out, P, ACT_NONE);
}

vt_status check_loaded(const vt_handle* h) {
  if (!h) return fail(VT_ERR_INVALID_ARG, "handle is NULL");
  if (!h->loaded) return fail(VT_ERR_NOT_LOADED, "weights are not loaded");
  return VT_OK;
}

}  // namespace

extern "C" {

const char* vt_last_error(void) { return g_last_error.c_str(); }

vt_status vt_create(const vt_config* cfg, vt_handle** out) {
  if (!cfg || !out) return fail(VT_ERR_INVALID_ARG, "cfg and out must not be NULL");
  const vt_config& c = *cfg;
  if (c.layers < 0 || c.hidden <= 0 || c.heads <= 0 || c.head_dim <= 0 || c.mlp <= 0 || c.patch <= 0 ||
      c.temporal_patch <= 0 || c.merge <= 0 || c.proj_hidden <= 0 || c.proj_out <= 0)
    return fail(VT_ERR_INVALID_ARG, "sizes must be positive");
  if (c.heads * c.head_dim != c.hidden)
    return fail(VT_ERR_INVALID_ARG, "heads * head_dim (%d * %d) != hidden (%d)", c.heads, c.head_dim, c.hidden);
  for (int a = 0; a < 3; ++a)
    if (c.rope_sections[a] < 0 || (c.rope_sections[a] & 1))
      return fail(VT_ERR_INVALID_ARG, "rope section %d must be even and non-negative", a);
  if (c.rope_sections[0] + c.rope_sections[1] + c.rope_sections[2] != c.head_dim)
    return fail(VT_ERR_INVALID_ARG, "rope sections must sum to head_dim");
  if (c.rope_sections[0] / 2 > kRopePairs || c.rope_sections[1] / 2 > kRopePairs || c.rope_sections[2] / 2 > kRopePairs)
    return fail(VT_ERR_UNSUPPORTED, "rope section wider than %d channels", 2 * kRopePairs);
  if (!(c.rope_theta > 0.f) || !(c.ln_eps > 0.f)) return fail(VT_ERR_INVALID_ARG, "rope_theta and ln_eps must be > 0");
  if (c.merge != 2) return fail(VT_ERR_UNSUPPORTED, "only a 2x2 merge is supported");
  if (!qkv_layout_supported(c))
    return fail(VT_ERR_UNSUPPORTED, "head_dim %d with sections %d/%d/%d has no fused QKV kernel", c.head_dim,
                c.rope_sections[0], c.rope_sections[1], c.rope_sections[2]);
  if (c.hidden % 8 || c.mlp % 8 || c.proj_hidden % 8 || c.proj_out % 8)
    return fail(VT_ERR_UNSUPPORTED, "widths must be multiples of 8");
  vt_handle* h = new vt_handle();
  h->cfg = c;
  *out = h;
  return VT_OK;
}

vt_status vt_destroy(vt_handle* h) {
  if (!h) return VT_OK;
  if (h->qkv_pack || h->rope_tab || h->bwd_pack) cudaDeviceSynchronize();
  if (h->qkv_pack) cudaFree(h->qkv_pack);
  if (h->bwd_pack) cudaFree(h->bwd_pack);
  if (h->rope_tab) cudaFree(h->rope_tab);
  delete h;
  return VT_OK;
}

vt_status vt_workspace_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* out) {
  if (!h || !out) return fail(VT_ERR_INVALID_ARG, "handle and out must not be NULL");
  int t, gh, gw;
  vt_status s = check_grid(h, B, grid_thw, &t, &gh, &gw);
  if (s) return s;
  *out = make_plan(h->cfg, B, t, gh, gw).total;
  return VT_OK;
}

vt_status vt_load_weights(vt_handle* h, const vt_weight* w, int n) {
  if (!h || (!w && n > 0) || n < 0) return fail(VT_ERR_INVALID_ARG, "bad arguments");
  const vt_config& c = h->cfg;
  std::map<std::string, const vt_weight*> byname;
  for (int i = 0; i < n; ++i) {
    if (!w[i].name || !w[i].data) return fail(VT_ERR_WEIGHT, "weight %d has a NULL name or data", i);
    if (!aligned16(w[i].data)) return fail(VT_ERR_WEIGHT, "%s is not 16-byte aligned", w[i].name);
    if (!byname.emplace(w[i].name, &w[i]).second) return fail(VT_ERR_WEIGHT, "duplicate weight %s", w[i].name);
  }
  std::map<std::string, bool> used;
  auto get = [&](const std::string& name, std::vector<int64_t> shape, const void** dst) -> vt_status {
    auto it = byname.find(name);
    if (it == byname.end()) return fail(VT_ERR_WEIGHT, "missing weight %s", name.c_str());
    const vt_weight& t = *it->second;
    bool ok = t.ndim == static_cast<int>(shape.size());
    for (size_t i = 0; ok && i < shape.size(); ++i) ok = t.shape[i] == shape[i];
    if (!ok) return fail(VT_ERR_WEIGHT, "weight %s has the wrong shape", name.c_str());
    used[name] = true;
    *dst = t.data;
    return VT_OK;
  };
  const int64_t d = c.hidden, m = c.mlp, P = c.proj_hidden, Po = c.proj_out;
  vt_status s;
  if ((s = get("embeddings.proj.weight", {d, 3, c.temporal_patch, c.patch, c.patch}, &h->pe_w))) return s;
  if ((s = get("embeddings.proj.bias", {d}, &h->pe_b))) return s;
  std::vector<vt_handle::Layer> layers(c.layers);
  std::vector<int> needs_pack;
  for (int i = 0; i < c.layers; ++i) {
    const std::string p = "layers." + std::to_string(i) + ".";
    vt_handle::Layer& L = layers[i];
    if ((s = get(p + "ln1.weight", {d}, &L.ln1_w)) || (s = get(p + "ln1.bias", {d}, &L.ln1_b)) ||
        (s = get(p + "ln2.weight", {d}, &L.ln2_w)) || (s = get(p + "ln2.bias", {d}, &L.ln2_b)) ||
        (s = get(p + "attn.o.weight", {d, d}, &L.o_w)) || (s = get(p + "attn.o.bias", {d}, &L.o_b)) ||
        (s = get(p + "mlp.fc1.weight", {m, d}, &L.fc1_w)) || (s = get(p + "mlp.fc1.bias", {m}, &L.fc1_b)) ||
        (s = get(p + "mlp.fc2.weight", {d, m}, &L.fc2_w)) || (s = get(p + "mlp.fc2.bias", {d}, &L.fc2_b)))
      return s;
    if (byname.count(p + "attn.qkv.weight")) {
      if ((s = get(p + "attn.qkv.weight", {3 * d, d}, &L.qkv_w)) || (s = get(p + "attn.qkv.bias", {3 * d}, &L.qkv_b)))
        return s;
    } else {
      needs_pack.push_back(i);
    }
  }
  if ((s = get("proj.patch_fc1.weight", {P, d}, &h->pa1_w)) || (s = get("proj.patch_fc1.bias", {P}, &h->pa1_b)) ||
      (s = get("proj.patch_fc2.weight", {P, P}, &h->pa2_w)) || (s = get("proj.patch_fc2.bias", {P}, &h->pa2_b)) ||
      (s = get("proj.merge_fc1.weight", {P, 4 * P}, &h->pb1_w)) || (s = get("proj.merge_fc1.bias", {P}, &h->pb1_b)) ||
      (s = get("proj.merge_fc2.weight", {Po, P}, &h->pb2_w)) || (s = get("proj.merge_fc2.bias", {Po}, &h->pb2_b)))
    return s;
  // Separate q, k, v: gather the pointers now, pack after every name is checked.
  std::vector<const void*> sep(needs_pack.size() * 6);
  for (size_t j = 0; j < needs_pack.size(); ++j) {
    const std::string p = "layers." + std::to_string(needs_pack[j]) + ".attn.";
    const char* parts[3] = {"q", "k", "v"};
    for (int a = 0; a < 3; ++a) {
      if ((s = get(p + parts[a] + ".weight", {d, d}, &sep[j * 6 + a])) ||
          (s = get(p + parts[a] + ".bias", {d}, &sep[j * 6 + 3 + a])))
        return s;
    }
  }
  for (auto& kv : byname)
    if (!used.count(kv.first)) return fail(VT_ERR_WEIGHT, "unknown weight %s", kv.first.c_str());

  // Device-side state: fused qkv packs and RoPE tables.  Transposed weights of an
  // earlier vt_enable_backward no longer match: drop them.
  if (h->bwd_pack) {
    cudaDeviceSynchronize();
    cudaFree(h->bwd_pack);
    h->bwd_pack = nullptr;
    h->layers_t.clear();
    h->pe_t = nullptr;
  }
  if (h->qkv_pack) {
    cudaFree(h->qkv_pack);
    h->qkv_pack = nullptr;
  }
  if (!needs_pack.empty()) {
    const size_t per = align256(3 * d * d * 2) + align256(3 * d * 2);
    cudaError_t e = cudaMalloc(&h->qkv_pack, per * needs_pack.size());
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(qkv pack)");
    for (size_t j = 0; j < needs_pack.size(); ++j) {
      char* base = static_cast<char*>(h->qkv_pack) + j * per;
      char* bias = base + align256(3 * d * d * 2);
      for (int a = 0; a < 3; ++a) {
        if ((e = cudaMemcpy(base + a * d * d * 2, sep[j * 6 + a], d * d * 2, cudaMemcpyDeviceToDevice)) ||
            (e = cudaMemcpy(bias + a * d * 2, sep[j * 6 + 3 + a], d * 2, cudaMemcpyDeviceToDevice)))
          return cuda_fail(e, "packing q/k/v");
      }
      layers[needs_pack[j]].qkv_w = base;
      layers[needs_pack[j]].qkv_b = bias;
    }
  }
  if (!h->rope_tab) {
    std::vector<float2> tab(static_cast<size_t>(3) * kRopeMaxPos * kRopePairs, make_float2(1.f, 0.f));
    for (int a = 0; a < 3; ++a) {
      const int sec = c.rope_sections[a];
      for (int pos = 0; pos < kRopeMaxPos; ++pos)
        for (int j = 0; j < sec / 2; ++j) {
          const double ang = pos * std::pow(static_cast<double>(c.rope_theta), -2.0 * j / sec);
          tab[(static_cast<size_t>(a) * kRopeMaxPos + pos) * kRopePairs + j] =
              make_float2(static_cast<float>(std::cos(ang)), static_cast<float>(std::sin(ang)));
        }
    }
    cudaError_t e = cudaMalloc(&h->rope_tab, tab.size() * sizeof(float2));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(rope tables)");
    if ((e = cudaMemcpy(h->rope_tab, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice)))
      return cuda_fail(e, "uploading rope tables");
  }
  h->layers = layers;
  h->loaded = true;
  return VT_OK;
}

// Everything after the patch vectors: patch-embed GEMM on the block-ordered patch
// vectors at ws + pl.unfold, the layers, the optional raster copy of the tower, the
// merge and projector.
static vt_status forward_embedded(vt_handle* h, int B, int t, int gh, int gw, void* out, void* tower_out, char* w,
                                  const Plan& pl, cudaStream_t st) {
  const vt_config& c = h->cfg;
  void* x = w + pl.x;
  vt_status s;
  if ((s = run_patch_embed(h, w + pl.unfold, x, w, pl, st))) return s;
  for (int i = 0; i < c.layers; ++i)
    if ((s = run_layer(h, i, x, x, B, t, gh, gw, ORDER_BLOCK, w, pl, st))) return s;
  if (tower_out) {
    ProfScope ps(CLS_REORDER, 0, 4.0 * pl.M * c.hidden, st);
    cudaError_t e = launch_reorder_rows(x, tower_out, B, t, gh, gw, c.hidden, 0, st);
    if (e != cudaSuccess) return cuda_fail(e, "reorder launch");
  }
  return run_projector(h, x, out, w, pl, st);
}

// Forward of B clips of F frames [B, F, 3, H, W] with grid (t, gh, gw), t = ceil(F / tp)
// (a still image is F = 1, t = 1).  Arguments are checked by the callers.
static vt_status forward_clips(vt_handle* h, const float* pixels, int F, int B, int t, int gh, int gw, void* out,
                               void* tower_out, void* ws, size_t ws_bytes, cudaStream_t st) {
  const vt_config& c = h->cfg;
  const Plan pl = make_plan(c, B, t, gh, gw);
  if (ws_bytes < pl.total)
    return fail(VT_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, pl.total);
  char* w = static_cast<char*>(ws);
  const int K0 = 3 * c.temporal_patch * c.patch * c.patch;
  {
    const double px_bytes = 4.0 * B * F * 3.0 * (gh * c.patch) * (gw * c.patch);
    ProfScope ps(CLS_UNFOLD, 0, px_bytes + 2.0 * pl.M * K0, st);
    cudaError_t e = launch_patch_unfold_frames(pixels, w + pl.unfold, B, F, gh * c.patch, gw * c.patch, c.patch,
                                               c.temporal_patch, ORDER_BLOCK, st);
    if (e != cudaSuccess) return cuda_fail(e, "patch unfold launch");
  }
  return forward_embedded(h, B, t, gh, gw, out, tower_out, w, pl, st);
}

static vt_status check_forward_ptrs(const float* pixels, const void* out, const void* tower_out, const void* ws) {
  if (!pixels || !out || !ws) return fail(VT_ERR_INVALID_ARG, "pixels, out and ws must not be NULL");
  if (!aligned16(pixels) || !aligned16(out) || !aligned16(ws) || (tower_out && !aligned16(tower_out)))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return VT_OK;
}

vt_status vt_forward(vt_handle* h, const float* pixels, const int32_t* grid_thw, int B, void* out, void* tower_out,
                     void* ws, size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if ((s = check_forward_ptrs(pixels, out, tower_out, ws))) return s;
  int t, gh, gw;
  if ((s = check_grid(h, B, grid_thw, &t, &gh, &gw))) return s;
  if ((s = check_still(t, "vt_forward"))) return s;
  return forward_clips(h, pixels, 1, B, t, gh, gw, out, tower_out, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

vt_status vt_forward_video(vt_handle* h, const float* clips, int frames, const int32_t* grid_thw, int B, void* out,
                           void* tower_out, void* ws, size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if ((s = check_forward_ptrs(clips, out, tower_out, ws))) return s;
  if (frames <= 0) return fail(VT_ERR_INVALID_ARG, "a clip needs at least one frame (got %d)", frames);
  int t, gh, gw;
  if ((s = check_grid(h, B, grid_thw, &t, &gh, &gw))) return s;
  const int tp = h->cfg.temporal_patch;
  if (t != (frames + tp - 1) / tp)
    return fail(VT_ERR_SHAPE, "grid t = %d does not match %d frames at temporal patch %d (expected %d)", t, frames,
                tp, (frames + tp - 1) / tp);
  return forward_clips(h, clips, frames, B, t, gh, gw, out, tower_out, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// OpenAI CLIP image statistics, used when the caller passes no mean / std.
const float kClipMean[3] = {0.48145466f, 0.4578275f, 0.40821073f};
const float kClipStd[3] = {0.26862954f, 0.26130258f, 0.27577711f};

// Checks decoded-image sizes against the target grid and splits the batch into
// launch tables of at most kMaxVarlenImages images.
vt_status build_preproc(const vt_config& c, const int32_t* src_hw, int B, int gh, int gw, const float* mean,
                        const float* std_, std::vector<PreprocTable>* tabs, int* rows_cap, double* src_bytes) {
  if (!src_hw) return fail(VT_ERR_INVALID_ARG, "src_hw is NULL");
  const float* m = mean ? mean : kClipMean;
  const float* sd = std_ ? std_ : kClipStd;
  for (int ch = 0; ch < 3; ++ch)
    if (!(sd[ch] > 0.f) || !std::isfinite(m[ch]))
      return fail(VT_ERR_INVALID_ARG, "channel %d: std must be positive and mean finite", ch);
  const int H1 = gh * c.patch, W1 = gw * c.patch;
  tabs->clear();
  long long off = 0;
  size_t cap = 1;
  for (int b = 0; b < B; ++b) {
    const int H0 = src_hw[2 * b], W0 = src_hw[2 * b + 1];
    if (H0 <= 0 || W0 <= 0) return fail(VT_ERR_INVALID_ARG, "image %d has size %dx%d", b, H0, W0);
    if (H0 > kMaxShrink * H1 || W0 > kMaxShrink * W1)
      return fail(VT_ERR_SHAPE, "image %d (%dx%d) is more than %dx the %dx%d target", b, H0, W0, kMaxShrink, H1, W1);
    if (b % kMaxVarlenImages == 0) {
      tabs->emplace_back();
      PreprocTable& t = tabs->back();
      std::memset(&t, 0, sizeof(t));
      for (int ch = 0; ch < 3; ++ch) {
        t.mean[ch] = m[ch];
        t.std[ch] = sd[ch];
      }
      off = 0;  // offsets are relative to the table's first image
    }
    PreprocTable& t = tabs->back();
    t.src_off[t.count] = off;
    t.src_h[t.count] = H0;
    t.src_w[t.count] = W0;
    ++t.count;
    off += 3ll * H0 * W0;
    *src_bytes += 3.0 * H0 * W0;
    cap = std::max(cap, preprocess_rows_bound(H0, H1, c.patch));
  }
  *rows_cap = static_cast<int>(cap);
  return VT_OK;
}

// Launches the tables one after the other; images and out advance per table.
vt_status run_preproc(const vt_config& c, const uint8_t* images, const std::vector<PreprocTable>& tabs, void* out,
                      int gh, int gw, int to_patches, int rows_cap, cudaStream_t st) {
  const size_t per_image = to_patches ? static_cast<size_t>(gh) * gw * 3 * c.temporal_patch * c.patch * c.patch * 2
                                      : static_cast<size_t>(3) * gh * c.patch * gw * c.patch * 4;
  char* o = static_cast<char*>(out);
  for (const PreprocTable& t : tabs) {
    cudaError_t e = launch_preprocess(images, t, o, gh, gw, c.patch, c.temporal_patch, ORDER_BLOCK, to_patches,
                                      rows_cap, st);
    if (e != cudaSuccess) return cuda_fail(e, "preprocess launch");
    images += t.src_off[t.count - 1] + 3ll * t.src_h[t.count - 1] * t.src_w[t.count - 1];
    o += per_image * t.count;
  }
  return VT_OK;
}

}  // namespace

extern "C" {

vt_status vt_preprocess(const vt_handle* h, const uint8_t* images, const int32_t* src_hw, int B,
                        const int32_t* grid_thw, const float* mean, const float* std_, float* pixels, void* stream) {
  if (!h) return fail(VT_ERR_INVALID_ARG, "handle is NULL");
  if (!images || !pixels) return fail(VT_ERR_INVALID_ARG, "images and pixels must not be NULL");
  if (!aligned16(pixels)) return fail(VT_ERR_INVALID_ARG, "pixels must be 16-byte aligned");
  int t, gh, gw;
  vt_status s = check_grid(h, B, grid_thw, &t, &gh, &gw);
  if (s) return s;
  if ((s = check_still(t, "vt_preprocess"))) return s;
  std::vector<PreprocTable> tabs;
  int cap;
  double src_bytes = 0;
  if ((s = build_preproc(h->cfg, src_hw, B, gh, gw, mean, std_, &tabs, &cap, &src_bytes))) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope ps(CLS_UNFOLD, 0, src_bytes + 4.0 * B * 3.0 * gh * gw * h->cfg.patch * h->cfg.patch, st);
  return run_preproc(h->cfg, images, tabs, pixels, gh, gw, 0, cap, st);
}

vt_status vt_forward_u8(vt_handle* h, const uint8_t* images, const int32_t* src_hw, int B, const int32_t* grid_thw,
                        const float* mean, const float* std_, void* out, void* tower_out, void* ws, size_t ws_bytes,
                        void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!images || !out || !ws) return fail(VT_ERR_INVALID_ARG, "images, out and ws must not be NULL");
  if (!aligned16(out) || !aligned16(ws) || (tower_out && !aligned16(tower_out)))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int t, gh, gw;
  if ((s = check_grid(h, B, grid_thw, &t, &gh, &gw))) return s;
  if ((s = check_still(t, "vt_forward_u8"))) return s;
  const vt_config& c = h->cfg;
  const Plan pl = make_plan(c, B, t, gh, gw);
  if (ws_bytes < pl.total)
    return fail(VT_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, pl.total);
  std::vector<PreprocTable> tabs;
  int cap;
  double src_bytes = 0;
  if ((s = build_preproc(c, src_hw, B, gh, gw, mean, std_, &tabs, &cap, &src_bytes))) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  {
    ProfScope ps(CLS_UNFOLD, 0, src_bytes + 2.0 * pl.M * 3 * c.temporal_patch * c.patch * c.patch, st);
    if ((s = run_preproc(c, images, tabs, w + pl.unfold, gh, gw, 1, cap, st))) return s;
  }
  return forward_embedded(h, B, t, gh, gw, out, tower_out, w, pl, st);
}

}  // extern "C"

namespace {

// Validates the grids of a variable-resolution batch and builds its table and plan.
vt_status build_varlen(const vt_handle* h, int B, const int32_t* grids, VarlenTable* vl, Plan* pl) {
  if (!grids) return fail(VT_ERR_INVALID_ARG, "grids is NULL");
  if (B <= 0 || B > kMaxVarlenImages)
    return fail(VT_ERR_INVALID_ARG, "a variable-resolution batch holds 1 to %d images (got %d)", kMaxVarlenImages, B);
  const vt_config& c = h->cfg;
  std::memset(vl, 0, sizeof(*vl));
  vl->count = B;
  long long tok = 0, pix = 0;
  int nmax = 0;
  for (int b = 0; b < B; ++b) {
    int t, gh, gw;
    vt_status s = check_grid(h, 1, grids + 3 * b, &t, &gh, &gw);
    if (s) return s;
    if ((s = check_still(t, "vt_forward_varlen"))) return s;
    const long long n = static_cast<long long>(gh) * gw;
    vl->tok_off[b] = static_cast<int>(tok);
    vl->gh[b] = gh;
    vl->gw[b] = gw;
    vl->pix_off[b] = pix;
    nmax = std::max(nmax, static_cast<int>(n));
    tok += n;
    pix += 3 * n * c.patch * c.patch;
    if (tok * c.heads > (1ll << 30)) return fail(VT_ERR_SHAPE, "too many tokens in one call");
  }
  vl->tok_off[B] = static_cast<int>(tok);
  // v^T of every image uses one stride (the largest image's tokens, rounded up to 8) so
  // that a single attention launch covers the batch; the padding is zeroed per forward.
  const int ld = round8(nmax);
  long long vt_elems = 0;
  for (int b = 0; b < B; ++b) {
    vl->ld_vt[b] = ld;
    vl->vt_off[b] = vt_elems;
    vt_elems += static_cast<long long>(c.heads) * c.head_dim * ld;
  }
  *pl = make_plan_core(c, static_cast<int>(tok), static_cast<size_t>(vt_elems));
  return VT_OK;
}

}  // namespace

extern "C" {

vt_status vt_workspace_bytes_varlen(const vt_handle* h, int B, const int32_t* grids, size_t* out) {
  if (!h || !out) return fail(VT_ERR_INVALID_ARG, "handle and out must not be NULL");
  VarlenTable vl;
  Plan pl;
  vt_status s = build_varlen(h, B, grids, &vl, &pl);
  if (s) return s;
  *out = pl.total;
  return VT_OK;
}

vt_status vt_forward_varlen(vt_handle* h, const float* pixels, const int32_t* grids, int B, void* out,
                            void* tower_out, void* ws, size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!pixels || !out || !ws) return fail(VT_ERR_INVALID_ARG, "pixels, out and ws must not be NULL");
  if (!aligned16(pixels) || !aligned16(out) || !aligned16(ws) || (tower_out && !aligned16(tower_out)))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  VarlenTable vl;
  Plan pl;
  if ((s = build_varlen(h, B, grids, &vl, &pl))) return s;
  if (ws_bytes < pl.total)
    return fail(VT_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, pl.total);
  const vt_config& c = h->cfg;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  void* x = w + pl.x;
  const int K0 = 3 * c.temporal_patch * c.patch * c.patch;
  {
    ProfScope ps(CLS_UNFOLD, 0, pl.M * (4.0 * 3 * c.patch * c.patch + 2.0 * K0), st);
    cudaError_t e = launch_patch_unfold_varlen(pixels, w + pl.unfold, vl, c.patch, c.temporal_patch, st);
    if (e != cudaSuccess) return cuda_fail(e, "patch unfold launch");
  }
  if ((s = run_patch_embed(h, w + pl.unfold, x, w, pl, st))) return s;
  // The QKV epilogue writes only each image's own v^T columns; the rest of the common
  // stride must read as zeros in the attention's P.V (P is zero there).
  {
    const size_t vt_bytes = static_cast<size_t>(B) * c.heads * c.head_dim * vl.ld_vt[0] * 2;
    cudaError_t e = cudaMemsetAsync(w + pl.vt, 0, vt_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing v^T padding");
  }
  for (int i = 0; i < c.layers; ++i)
    if ((s = run_layer(h, i, x, x, B, 1, 0, 0, ORDER_BLOCK, w, pl, st, &vl))) return s;
  if (tower_out) {
    for (int b = 0; b < B; ++b) {
      ProfScope ps(CLS_REORDER, 0, 4.0 * (vl.tok_off[b + 1] - vl.tok_off[b]) * c.hidden, st);
      const size_t off = static_cast<size_t>(vl.tok_off[b]) * c.hidden * 2;
      cudaError_t e = launch_reorder_rows(static_cast<char*>(x) + off, static_cast<char*>(tower_out) + off, 1, 1,
                                          vl.gh[b], vl.gw[b], c.hidden, 0, st);
      if (e != cudaSuccess) return cuda_fail(e, "reorder launch");
    }
  }
  // Each image's tokens start at a multiple of 4 and keep their 2x2 groups together,
  // so the merged [tokens/4, 4P] view spans the whole packed batch.
  return run_projector(h, x, out, w, pl, st);
}

vt_status vt_forward_host_workspace_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* out) {
  size_t base;
  vt_status s = vt_workspace_bytes(h, B, grid_thw, &base);
  if (s) return s;
  if ((s = check_still(grid_thw[0], "vt_forward_host"))) return s;
  const vt_config& c = h->cfg;
  const size_t N = static_cast<size_t>(grid_thw[0]) * grid_thw[1] * grid_thw[2];
  const size_t px = static_cast<size_t>(B) * 3 * N * c.patch * c.patch * 4;
  const size_t o = static_cast<size_t>(B) * (N / 4) * c.proj_out * 2;
  *out = align256(base) + align256(px) + align256(o);
  return VT_OK;
}

// vt_forward_host without the final synchronisation (see include/vt.h).
static vt_status forward_host(vt_handle* h, const float* pixels_host, const int32_t* grid_thw, int B, void* out_host,
                              void* ws, size_t ws_bytes, void* stream, bool sync);

vt_status vt_forward_host(vt_handle* h, const float* pixels_host, const int32_t* grid_thw, int B, void* out_host,
                          void* ws, size_t ws_bytes, void* stream) {
  return forward_host(h, pixels_host, grid_thw, B, out_host, ws, ws_bytes, stream, true);
}

vt_status vt_forward_host_async(vt_handle* h, const float* pixels_host, const int32_t* grid_thw, int B,
                                void* out_host, void* ws, size_t ws_bytes, void* stream) {
  return forward_host(h, pixels_host, grid_thw, B, out_host, ws, ws_bytes, stream, false);
}

static vt_status forward_host(vt_handle* h, const float* pixels_host, const int32_t* grid_thw, int B, void* out_host,
                              void* ws, size_t ws_bytes, void* stream, bool sync) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!pixels_host || !out_host || !ws) return fail(VT_ERR_INVALID_ARG, "pixels, out and ws must not be NULL");
  size_t need, base;
  if ((s = vt_forward_host_workspace_bytes(h, B, grid_thw, &need))) return s;
  if (ws_bytes < need) return fail(VT_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, need);
  vt_workspace_bytes(h, B, grid_thw, &base);
  const vt_config& c = h->cfg;
  const size_t N = static_cast<size_t>(grid_thw[0]) * grid_thw[1] * grid_thw[2];
  const size_t px = static_cast<size_t>(B) * 3 * N * c.patch * c.patch * 4;
  const size_t o = static_cast<size_t>(B) * (N / 4) * c.proj_out * 2;
  char* w = static_cast<char*>(ws);
  float* dpx = reinterpret_cast<float*>(w + align256(base));
  char* dout = w + align256(base) + align256(px);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(dpx, pixels_host, px, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e, "copying pixels to the device");
  if ((s = vt_forward(h, dpx, grid_thw, B, dout, nullptr, ws, base, stream))) return s;
  if ((e = cudaMemcpyAsync(out_host, dout, o, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail(e, "copying the output to the host");
  if (sync && (e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "stream synchronisation");
  return VT_OK;
}

vt_status vt_tower_layer(vt_handle* h, int layer, const void* x_in, void* x_out, const int32_t* grid_thw, int B,
                         void* ws, size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (layer < 0 || layer >= h->cfg.layers) return fail(VT_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (!x_in || !x_out || !ws) return fail(VT_ERR_INVALID_ARG, "x_in, x_out and ws must not be NULL");
  if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(ws))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int t, gh, gw;
  if ((s = check_grid(h, B, grid_thw, &t, &gh, &gw))) return s;
  const Plan pl = make_plan(h->cfg, B, t, gh, gw);
  if (ws_bytes < pl.total) return fail(VT_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, pl.total);
  return run_layer(h, layer, x_in, x_out, B, t, gh, gw, ORDER_RASTER, static_cast<char*>(ws), pl,
                   static_cast<cudaStream_t>(stream));
}

vt_status vt_patch_embed(vt_handle* h, const float* pixels, const int32_t* grid_thw, int B, void* x_out, void* ws,
                         size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!pixels || !x_out || !ws) return fail(VT_ERR_INVALID_ARG, "pixels, x_out and ws must not be NULL");
  int t, gh, gw;
  if ((s = check_grid(h, B, grid_thw, &t, &gh, &gw))) return s;
  if ((s = check_still(t, "vt_patch_embed"))) return s;
  const vt_config& c = h->cfg;
  const Plan pl = make_plan(c, B, t, gh, gw);
  if (ws_bytes < pl.total) return fail(VT_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, pl.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  cudaError_t e = launch_patch_unfold(pixels, w + pl.unfold, B, gh * c.patch, gw * c.patch, c.patch, c.temporal_patch,
                                      ORDER_RASTER, st);
  if (e != cudaSuccess) return cuda_fail(e, "patch unfold launch");
  return run_patch_embed(h, w + pl.unfold, x_out, w, pl, st);
}

vt_status vt_merge_project(vt_handle* h, const void* tower, const int32_t* grid_thw, int B, void* out, void* ws,
                           size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!tower || !out || !ws) return fail(VT_ERR_INVALID_ARG, "tower, out and ws must not be NULL");
  if (!aligned16(tower) || !aligned16(out) || !aligned16(ws))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int t, gh, gw;
  if ((s = check_grid(h, B, grid_thw, &t, &gh, &gw))) return s;
  const Plan pl = make_plan(h->cfg, B, t, gh, gw);
  if (ws_bytes < pl.total) return fail(VT_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, pl.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  {
    ProfScope ps(CLS_REORDER, 0, 4.0 * pl.M * h->cfg.hidden, st);
    cudaError_t e = launch_reorder_rows(tower, w + pl.x, B, t, gh, gw, h->cfg.hidden, 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "reorder launch");
  }
  return run_projector(h, w + pl.x, out, w, pl, st);
}

vt_status vt_attention_workspace_bytes(int B, int H, int N, int D, size_t* out) {
  if (!out || B <= 0 || H <= 0 || N <= 0 || D <= 0) return fail(VT_ERR_INVALID_ARG, "bad arguments");
  const size_t ldv = static_cast<size_t>(round8(N));
  *out = 3 * align256(static_cast<size_t>(B) * H * D * ldv * 2);
  return VT_OK;
}

vt_status vt_attention_prepared(const void* q, const void* k, const void* vt_, int ld_vt, void* o, int B, int H, int N,
                                int D, float scale, void* stream) {
  vt_status s = check_attention_dims(B, H, N, D, scale);
  if (s) return s;
  if (!q || !k || !vt_ || !o) return fail(VT_ERR_INVALID_ARG, "NULL operand");
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt_) || !aligned16(o))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (ld_vt < N || (ld_vt % 8)) return fail(VT_ERR_INVALID_ARG, "ld_vt must be >= N and a multiple of 8");
  AttnParams a{q, k, vt_, o, B, H, N, D, ld_vt, scale};
  return run_attention(a, static_cast<cudaStream_t>(stream));
}

vt_status vt_attention(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                       const int32_t* pos_thw, const int32_t* sections, float theta, float scale, void* ws,
                       size_t ws_bytes, void* stream) {
  vt_status s = check_attention_dims(B, H, N, D, scale);
  if (s) return s;
  if (!q || !k || !v || !o || !ws) return fail(VT_ERR_INVALID_ARG, "NULL operand or workspace");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ws))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int sec[3] = {0, 0, 0};
  if (pos_thw) {
    if (!sections) return fail(VT_ERR_INVALID_ARG, "sections must be given with pos_thw");
    for (int a = 0; a < 3; ++a) {
      sec[a] = sections[a];
      if (sec[a] < 0 || (sec[a] & 1)) return fail(VT_ERR_INVALID_ARG, "rope sections must be even");
    }
    if (sec[0] + sec[1] + sec[2] != D) return fail(VT_ERR_INVALID_ARG, "rope sections must sum to head_dim");
    if (!(theta > 0.f)) return fail(VT_ERR_INVALID_ARG, "theta must be positive");
  }
  size_t need;
  vt_attention_workspace_bytes(B, H, N, D, &need);
  if (ws_bytes < need) return fail(VT_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, need);
  const int ldv = round8(N);
  const size_t part = align256(static_cast<size_t>(B) * H * D * ldv * 2);
  char* w = static_cast<char*>(ws);
  void* qr = w;
  void* kr = w + part;
  void* vt_ = w + 2 * part;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = run_attention_prep(q, k, v, qr, kr, vt_, B, H, N, D, ldv, pos_thw, sec, theta, st))) return s;
  AttnParams a{qr, kr, vt_, o, B, H, N, D, ldv, scale};
  return run_attention(a, st);
}

vt_status vt_linear(const void* A, const void* W, const void* bias, const void* resid, void* out, int M, int N, int K,
                    int act, void* stream) {
  if (!A || !W || !out) return fail(VT_ERR_INVALID_ARG, "A, W and out must not be NULL");
  if (M <= 0 || N <= 0 || K <= 0) return fail(VT_ERR_INVALID_ARG, "M, N, K must be positive");
  if (N % 8 || K % 8) return fail(VT_ERR_INVALID_ARG, "N and K must be multiples of 8");
  if (act < 0 || act > 2) return fail(VT_ERR_INVALID_ARG, "act must be 0, 1 or 2");
  if (!aligned16(A) || !aligned16(W) || !aligned16(out) || (bias && !aligned16(bias)) || (resid && !aligned16(resid)))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return run_gemm(gemm_params(A, K, W, K, bias, resid, N, out, N, M, N, K, act), static_cast<cudaStream_t>(stream));
}

vt_status vt_linear_ws(const void* A, const void* W, const void* bias, const void* resid, void* out, int M, int N,
                       int K, int act, void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < gemm_split_bytes()) return vt_linear(A, W, bias, resid, out, M, N, K, act, stream);
  if (!aligned16(ws)) return fail(VT_ERR_INVALID_ARG, "ws must be 16-byte aligned");
  if (!A || !W || !out) return fail(VT_ERR_INVALID_ARG, "A, W and out must not be NULL");
  if (M <= 0 || N <= 0 || K <= 0) return fail(VT_ERR_INVALID_ARG, "M, N, K must be positive");
  if (N % 8 || K % 8) return fail(VT_ERR_INVALID_ARG, "N and K must be multiples of 8");
  if (act < 0 || act > 2) return fail(VT_ERR_INVALID_ARG, "act must be 0, 1 or 2");
  if (!aligned16(A) || !aligned16(W) || !aligned16(out) || (bias && !aligned16(bias)) || (resid && !aligned16(resid)))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return run_gemm(split_k(gemm_params(A, K, W, K, bias, resid, N, out, N, M, N, K, act), static_cast<char*>(ws)),
                  static_cast<cudaStream_t>(stream));
}

vt_status vt_linear_workspace_bytes(size_t* out) {
  if (!out) return fail(VT_ERR_INVALID_ARG, "out is NULL");
  *out = gemm_split_bytes();
  return VT_OK;
}

vt_status vt_layernorm(const void* x, const void* gamma, const void* beta, void* y, int rows, int cols, float eps,
                       void* stream) {
  if (!x || !gamma || !beta || !y) return fail(VT_ERR_INVALID_ARG, "NULL operand");
  if (rows <= 0 || cols <= 0 || !(eps > 0.f)) return fail(VT_ERR_INVALID_ARG, "rows, cols, eps must be positive");
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(beta) || !aligned16(y) || cols % 8)
    return fail(VT_ERR_INVALID_ARG, "16-byte aligned rows required (cols multiple of 8)");
  return run_layernorm(x, gamma, beta, y, rows, cols, eps, static_cast<cudaStream_t>(stream));
}

vt_status vt_patch_unfold(const float* pixels, void* out, int B, int H, int W, int patch, int temporal_patch, int order,
                          void* stream) {
  if (!pixels || !out) return fail(VT_ERR_INVALID_ARG, "NULL operand");
  if (B <= 0 || H <= 0 || W <= 0 || patch <= 0 || temporal_patch <= 0)
    return fail(VT_ERR_INVALID_ARG, "sizes must be positive");
  if (H % patch || W % patch) return fail(VT_ERR_SHAPE, "image side not a multiple of the patch");
  if (order != ORDER_RASTER && order != ORDER_BLOCK) return fail(VT_ERR_INVALID_ARG, "order must be 0 or 1");
  if (order == ORDER_BLOCK && ((H / patch) % 2 || (W / patch) % 2))
    return fail(VT_ERR_SHAPE, "block order needs an even grid");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const double rows = static_cast<double>(B) * (H / patch) * (W / patch);
  ProfScope ps(CLS_UNFOLD, 0, rows * (4.0 * 3 * patch * patch + 2.0 * 3 * temporal_patch * patch * patch), st);
  cudaError_t e = launch_patch_unfold(pixels, out, B, H, W, patch, temporal_patch, order, st);
  if (e != cudaSuccess) return cuda_fail(e, "patch unfold launch");
  return VT_OK;
}

vt_status vt_index_maps(const int32_t* g, int32_t* token_order, int32_t* pos_thw, int32_t* merge_src) {
  if (!g) return fail(VT_ERR_INVALID_ARG, "grid_thw is NULL");
  const int t = g[0], gh = g[1], gw = g[2];
  if (t <= 0 || gh <= 0 || gw <= 0) return fail(VT_ERR_INVALID_ARG, "grid must be positive");
  if (gh % 2 || gw % 2) return fail(VT_ERR_SHAPE, "grid must be even for the 2x2 merge");
  const int N = t * gh * gw;
  for (int n = 0; n < N; ++n) {
    int tt, hh, ww;
    token_position(n, gh, gw, ORDER_BLOCK, &tt, &hh, &ww);
    const int raster = (tt * gh + hh) * gw + ww;
    if (token_order) token_order[n] = raster;
    if (merge_src) merge_src[(n / 4) * 4 + (n % 4)] = raster;
    int rt, rh, rw;
    token_position(n, gh, gw, ORDER_RASTER, &rt, &rh, &rw);
    if (pos_thw) {
      pos_thw[3 * n + 0] = rt;
      pos_thw[3 * n + 1] = rh;
      pos_thw[3 * n + 2] = rw;
    }
  }
  return VT_OK;
}

vt_status vt_check(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronisation");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending launch error");
  const unsigned int ge = gemm_read_clear_error(st);
  const unsigned int ae = attention_read_clear_error(st);
  const unsigned int se = selftest_read_clear_error(st);
  const unsigned int pe = preprocess_read_clear_error(st);
  const unsigned int be = attention_bwd_read_clear_error(st);
  if (ge || ae || se || be)
    return fail(VT_ERR_TIMEOUT,
                "kernel wait limit reached (gemm flags %u, attention flags %u, attention backward flags %u, "
                "self-test flags %u)",
                ge, ae, be, se);
  if (pe) return fail(VT_ERR_CUDA, "preprocess tap window above its bound (flags %u): results are wrong", pe);
  return VT_OK;
}

vt_status vt_profile_begin(void* stream) {
  (void)stream;
  std::lock_guard<std::mutex> l(g_prof.mu);
  for (auto& r : g_prof.recs) {
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.recs.clear();
  g_prof.done.clear();
  for (int c = 0; c < CLS_COUNT; ++c) {
    g_prof.ms[c] = g_prof.flops[c] = g_prof.bytes[c] = 0;
    g_prof.n[c] = 0;
  }
  g_prof.on = true;
  return VT_OK;
}

vt_status vt_profile_end(void* stream) {
  (void)stream;
  std::lock_guard<std::mutex> l(g_prof.mu);
  g_prof.on = false;
  return VT_OK;
}

namespace {
// Resolves the pending event pairs into per-launch records and class totals.
vt_status resolve_profile() {
  for (auto& r : g_prof.recs) {
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile event");
    float t = 0;
    cudaEventElapsedTime(&t, r.a, r.b);
    g_prof.ms[r.cls] += t;
    g_prof.flops[r.cls] += r.flops;
    g_prof.bytes[r.cls] += r.bytes;
    g_prof.n[r.cls] += r.kernels;
    g_prof.done.push_back({r.cls, static_cast<double>(t), r.flops, r.bytes});
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.recs.clear();
  return VT_OK;
}
}  // namespace

vt_status vt_profile_read(int cls, double* ms, int64_t* launches, double* flops, double* bytes) {
  if (cls < 0 || cls >= CLS_COUNT) return fail(VT_ERR_INVALID_ARG, "class out of range");
  std::lock_guard<std::mutex> l(g_prof.mu);
  vt_status s = resolve_profile();
  if (s) return s;
  if (ms) *ms = g_prof.ms[cls];
  if (launches) *launches = g_prof.n[cls];
  if (flops) *flops = g_prof.flops[cls];
  if (bytes) *bytes = g_prof.bytes[cls];
  return VT_OK;
}

vt_status vt_profile_launches(int64_t* count) {
  if (!count) return fail(VT_ERR_INVALID_ARG, "count is NULL");
  std::lock_guard<std::mutex> l(g_prof.mu);
  vt_status s = resolve_profile();
  if (s) return s;
  *count = static_cast<int64_t>(g_prof.done.size());
  return VT_OK;
}

vt_status vt_profile_launch(int64_t i, int* cls, double* ms, double* flops, double* bytes) {
  std::lock_guard<std::mutex> l(g_prof.mu);
  if (i < 0 || i >= static_cast<int64_t>(g_prof.done.size())) return fail(VT_ERR_INVALID_ARG, "launch index out of range");
  const DoneRec& d = g_prof.done[static_cast<size_t>(i)];
  if (cls) *cls = d.cls;
  if (ms) *ms = d.ms;
  if (flops) *flops = d.flops;
  if (bytes) *bytes = d.bytes;
  return VT_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ backward
//
// Gradient of a loss with respect to the pixels, given its gradient with respect to the
// tower output: the reverse of every layer (from the activations its forward saved), then the
// patch embedding and the fold onto the image.  The derivative follows the chain rule
// through the forward of the "MiniMax-M3 Vision" model card (Architecture table); the
// "v2_loaders" findings (summary, section 3) describe the loaders as differentiable,
// their probe backpropagating the pooled tower feature to the image.

namespace {

// What the forward keeps of every layer for the backward (so that the backward runs no
// forward GEMM or attention again): the layer input, the rotated q and k, v^T, the
// attention output and its per-query log-sum-exp, the residual stream after attention,
// and the MLP pre-activation.  Offsets within one layer's block.
struct SavedLayout {
  int N, M, ld, lds;
  size_t x, q, k, vt, a, x1, z, lse, per_layer;
};

SavedLayout saved_layout(const vt_config& c, int B, int N) {
  SavedLayout L;
  L.N = N;
  L.M = B * N;
  L.ld = round8(N);
  L.lds = (N + 63) / 64 * 64;
  const size_t d = c.hidden, M = static_cast<size_t>(L.M);
  const size_t headT = static_cast<size_t>(B) * c.heads * c.head_dim * L.ld;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.x = take(M * d * 2);
  L.q = take(M * d * 2);
  L.k = take(M * d * 2);
  L.vt = take(headT * 2);
  L.a = take(M * d * 2);
  L.x1 = take(M * d * 2);
  L.z = take(M * static_cast<size_t>(c.mlp) * 2);
  L.lse = take(static_cast<size_t>(B) * c.heads * L.lds * 4);
  L.per_layer = off;
  return L;
}

// Backward workspace: the running gradient dx, scratch for the gradients of the LayerNorm
// outputs (dg, dh), the MLP gradient (also the patch-vector gradient at the end), dO,
// the [M, 3d] qkv gradient and the per-query delta.
struct BwdPlan {
  int N, M, ld, lds;
  size_t dx, xn, hmid, dO, dqkv, delta, sk, total;
};

BwdPlan make_bwd_plan(const vt_config& c, int B, int N) {
  BwdPlan p;
  p.N = N;
  p.M = B * N;
  p.ld = round8(N);
  p.lds = (N + 63) / 64 * 64;
  const size_t d = c.hidden, M = static_cast<size_t>(p.M);
  const size_t K0 = 3ull * c.temporal_patch * c.patch * c.patch;
  const size_t stats = static_cast<size_t>(B) * c.heads * p.lds;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  p.dx = take(M * d * 2);
  p.xn = take(M * d * 2);
  p.hmid = take(M * std::max<size_t>(c.mlp, K0) * 2);
  p.dO = take(M * d * 2);
  p.dqkv = take(M * 3 * d * 2);
  p.delta = take(stats * 4);
  p.sk = take(gemm_split_bytes());
  p.total = off;
  return p;
}

vt_status run_layernorm_backward(const void* x, const void* g, const void* dy, const void* dres, void* dx, int rows,
                                 int cols, float eps, cudaStream_t st) {
  ProfScope ps(CLS_BWD_MISC, 0, 8.0 * rows * static_cast<double>(cols), st);
  cudaError_t e = launch_layernorm_backward(x, g, dy, dres, dx, rows, cols, eps, st);
  if (e != cudaSuccess) return cuda_fail(e, "layernorm backward launch");
  return VT_OK;
}

vt_status run_attention_backward(const AttnBwdParams& p, cudaStream_t st) {
  // 5 matrix products per head (S, dP, dV, dK, dQ): 10 N^2 D
  ProfScope ps(CLS_ATTN_BWD, 10.0 * p.B * p.H * static_cast<double>(p.N) * p.N * p.D,
               2.0 * p.B * p.H * static_cast<double>(p.N) * p.D * 8, st);
  cudaError_t e = launch_attention_backward(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention backward launch");
  return VT_OK;
}

// One layer forward on block-ordered tokens that keeps what the backward needs in the
// layer's saved block `sv` (its input x is already there); writes the layer output to
// x_out.  Same kernels and arithmetic as run_layer.
vt_status run_layer_saving(vt_handle* h, int i, char* sv, const SavedLayout& sl, void* x_out, int B, int gh, int gw,
                           char* w, const Plan& pl, cudaStream_t st) {
  const vt_config& c = h->cfg;
  const vt_handle::Layer& L = h->layers[i];
  const int d = c.hidden, m = c.mlp, M = sl.M;
  void* xn = w + pl.xn;
  void* hmid = w + pl.hmid;
  vt_status s;
  if ((s = run_layernorm(sv + sl.x, L.ln1_w, L.ln1_b, xn, M, d, c.ln_eps, st))) return s;
  {
    GemmParams p = gemm_params(xn, d, L.qkv_w, d, L.qkv_b, nullptr, 0, nullptr, 0, M, 3 * d, d, ACT_NONE);
    p.q = sv + sl.q;
    p.k = sv + sl.k;
    p.vt = sv + sl.vt;
    p.heads = c.heads;
    p.head_dim = c.head_dim;
    p.ntok = sl.N;
    p.ld_vt = sl.ld;
    p.gt = 1;
    p.gh = gh;
    p.gw = gw;
    p.order = ORDER_BLOCK;
    p.rope = c.use_rope;
    for (int j = 0; j < 3; ++j) p.sections[j] = c.rope_sections[j];
    p.rope_tab = h->rope_tab;
    ProfScope ps(CLS_GEMM, 2.0 * M * 3.0 * d * d, 0, st);
    cudaError_t e = launch_gemm(p, st, 1);
    if (e != cudaSuccess) return cuda_fail(e, "qkv gemm launch");
  }
  {
    AttnParams a{};
    a.q = sv + sl.q;
    a.k = sv + sl.k;
    a.vt = sv + sl.vt;
    a.o = sv + sl.a;
    a.B = B;
    a.H = c.heads;
    a.N = sl.N;
    a.D = c.head_dim;
    a.ld_vt = sl.ld;
    a.scale = 1.0f / std::sqrt(static_cast<float>(c.head_dim));
    a.lse = reinterpret_cast<float*>(sv + sl.lse);
    a.ld_lse = sl.lds;
    if ((s = run_attention(a, st))) return s;
  }
  if ((s = run_gemm(
           split_k(gemm_params(sv + sl.a, d, L.o_w, d, L.o_b, sv + sl.x, d, sv + sl.x1, d, M, d, d, ACT_NONE), w + pl.sk),
           st)))
    return s;
  if ((s = run_layernorm(sv + sl.x1, L.ln2_w, L.ln2_b, xn, M, d, c.ln_eps, st))) return s;
  {
    GemmParams p = gemm_params(xn, d, L.fc1_w, d, L.fc1_b, nullptr, 0, hmid, m, M, m, d,
                               c.gelu_tanh ? ACT_GELU_TANH : ACT_GELU_ERF);
    p.pre_out = sv + sl.z;  // the pre-activation, for the GELU derivative
    if ((s = run_gemm(p, st))) return s;
  }
  return run_gemm(
      split_k(gemm_params(hmid, m, L.fc2_w, m, L.fc2_b, sv + sl.x1, d, x_out, d, M, d, m, ACT_NONE), w + pl.sk), st);
}

// One layer backward on block-ordered tokens: dx (in: d loss / d layer output; out:
// d loss / d layer input), from the layer's saved block.
vt_status run_layer_backward(vt_handle* h, int i, const char* sv, const SavedLayout& sl, int B, int gh, int gw,
                             char* w, const BwdPlan& bp, cudaStream_t st) {
  const vt_config& c = h->cfg;
  const vt_handle::Layer& L = h->layers[i];
  const vt_handle::LayerT& T = h->layers_t[i];
  const int d = c.hidden, m = c.mlp, M = bp.M, N = bp.N, H = c.heads, D = c.head_dim;
  void* dx = w + bp.dx;
  void* xn = w + bp.xn;
  void* hmid = w + bp.hmid;
  vt_status s;
  // ---- MLP branch: dz = (dx W2) * gelu'(z), dg = dz W1, dx += LN2^T(dg)
  const int dact = c.gelu_tanh ? ACT_DGELU_TANH : ACT_DGELU_ERF;
  if ((s = run_gemm(gemm_params(dx, d, T.fc2_t, d, nullptr, sv + sl.z, m, hmid, m, M, m, d, dact), st))) return s;
  if ((s = run_gemm(split_k(gemm_params(hmid, m, T.fc1_t, m, nullptr, nullptr, 0, xn, d, M, d, m, ACT_NONE), w + bp.sk),
                    st)))
    return s;
  if ((s = run_layernorm_backward(sv + sl.x1, L.ln2_w, xn, dx, dx, M, d, c.ln_eps, st))) return s;
  // ---- attention branch: dO = dx Wo, attention backward, dh = dqkv Wqkv, dx += LN1^T(dh)
  if ((s = run_gemm(
           split_k(gemm_params(dx, d, T.o_t, d, nullptr, nullptr, 0, w + bp.dO, d, M, d, d, ACT_NONE), w + bp.sk), st)))
    return s;
  {
    ProfScope ps(CLS_BWD_MISC, 0, 4.0 * M * d + 4.0 * M * H, st);
    cudaError_t e = launch_attention_delta(w + bp.dO, sv + sl.a, reinterpret_cast<float*>(w + bp.delta), B, N, H, D,
                                           bp.lds, st);
    if (e != cudaSuccess) return cuda_fail(e, "delta launch");
  }
  {
    AttnBwdParams a{};
    a.q = sv + sl.q;
    a.k = sv + sl.k;
    a.vt = sv + sl.vt;
    a.dO = w + bp.dO;
    a.lse = reinterpret_cast<const float*>(sv + sl.lse);
    a.delta = reinterpret_cast<const float*>(w + bp.delta);
    a.ld_stats = bp.lds;
    a.dqkv = w + bp.dqkv;
    a.ld_dqkv = 3 * d;
    a.B = B;
    a.H = H;
    a.N = N;
    a.D = D;
    a.ld = sl.ld;
    a.scale = 1.0f / std::sqrt(static_cast<float>(D));
    a.rope = c.use_rope;
    for (int j = 0; j < 3; ++j) a.sections[j] = c.rope_sections[j];
    a.rope_tab = h->rope_tab;
    a.gh = gh;
    a.gw = gw;
    a.order = ORDER_BLOCK;
    if ((s = run_attention_backward(a, st))) return s;
  }
  if ((s = run_gemm(split_k(gemm_params(w + bp.dqkv, 3 * d, T.qkv_t, 3 * d, nullptr, nullptr, 0, xn, d, M, d, 3 * d,
                                        ACT_NONE),
                            w + bp.sk),
                    st)))
    return s;
  return run_layernorm_backward(sv + sl.x, L.ln1_w, xn, dx, dx, M, d, c.ln_eps, st);
}

vt_status check_backward_grid(const vt_handle* h, int B, const int32_t* grid_thw, int* gh, int* gw) {
  int t;
  vt_status s = check_grid(h, B, grid_thw, &t, gh, gw);
  if (s) return s;
  if ((s = check_still(t, "the backward"))) return s;
  return VT_OK;
}

}  // namespace

extern "C" {

vt_status vt_enable_backward(vt_handle* h) {
  vt_status s = check_loaded(h);
  if (s) return s;
  const vt_config& c = h->cfg;
  if (!((c.head_dim == 80 && (!c.use_rope || (c.rope_sections[0] == 16 && c.rope_sections[1] == 32 &&
                                               c.rope_sections[2] == 32))) ||
        (c.head_dim == 32 && (!c.use_rope || (c.rope_sections[0] == 8 && c.rope_sections[1] == 12 &&
                                               c.rope_sections[2] == 12)))))
    return fail(VT_ERR_UNSUPPORTED, "the attention backward covers head_dim 80 (16/32/32) and 32 (8/12/12)");
  if (h->bwd_pack) return VT_OK;
  const size_t d = c.hidden, m = c.mlp, K0 = 3ull * c.temporal_patch * c.patch * c.patch;
  const size_t per_layer = align256(3 * d * d * 2) + align256(d * d * 2) + 2 * align256(d * m * 2);
  void* pack = nullptr;
  cudaError_t e = cudaMalloc(&pack, per_layer * c.layers + align256(K0 * d * 2));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(transposed weights)");
  std::vector<vt_handle::LayerT> lt(c.layers);
  char* base = static_cast<char*>(pack);
  for (int i = 0; i < c.layers && e == cudaSuccess; ++i) {
    vt_handle::LayerT& T = lt[i];
    const vt_handle::Layer& L = h->layers[i];
    T.qkv_t = base;
    T.o_t = base + align256(3 * d * d * 2);
    T.fc1_t = static_cast<char*>(T.o_t) + align256(d * d * 2);
    T.fc2_t = static_cast<char*>(T.fc1_t) + align256(d * m * 2);
    base += per_layer;
    // W [out, in] -> W^T [in, out]
    e = launch_transpose(L.qkv_w, T.qkv_t, 1, 1, 3 * d, d, 0, 0, d, 0, 0, 3 * d, 0);
    if (e == cudaSuccess) e = launch_transpose(L.o_w, T.o_t, 1, 1, d, d, 0, 0, d, 0, 0, d, 0);
    if (e == cudaSuccess) e = launch_transpose(L.fc1_w, T.fc1_t, 1, 1, m, d, 0, 0, d, 0, 0, m, 0);
    if (e == cudaSuccess) e = launch_transpose(L.fc2_w, T.fc2_t, 1, 1, d, m, 0, 0, m, 0, 0, d, 0);
  }
  void* pe_t = base;
  if (e == cudaSuccess) e = launch_transpose(h->pe_w, pe_t, 1, 1, d, K0, 0, 0, K0, 0, 0, d, 0);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(pack);
    return cuda_fail(e, "transposing weights");
  }
  h->layers_t = std::move(lt);
  h->pe_t = pe_t;
  h->bwd_pack = pack;
  return VT_OK;
}

vt_status vt_backward_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* saved_bytes,
                            size_t* ws_bytes) {
  if (!h || !saved_bytes || !ws_bytes) return fail(VT_ERR_INVALID_ARG, "handle and outputs must not be NULL");
  int gh, gw;
  vt_status s = check_backward_grid(h, B, grid_thw, &gh, &gw);
  if (s) return s;
  const vt_config& c = h->cfg;
  *saved_bytes = static_cast<size_t>(c.layers) * saved_layout(c, B, gh * gw).per_layer;
  *ws_bytes = std::max(make_plan(c, B, 1, gh, gw).total, make_bwd_plan(c, B, gh * gw).total);
  return VT_OK;
}

vt_status vt_forward_saved(vt_handle* h, const float* pixels, const int32_t* grid_thw, int B, void* tower_out,
                           void* saved, size_t saved_bytes, void* ws, size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!pixels || !tower_out || !saved || !ws) return fail(VT_ERR_INVALID_ARG, "pointers must not be NULL");
  if (!aligned16(pixels) || !aligned16(tower_out) || !aligned16(saved) || !aligned16(ws))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int gh, gw;
  if ((s = check_backward_grid(h, B, grid_thw, &gh, &gw))) return s;
  size_t need_saved, need_ws;
  vt_backward_bytes(h, B, grid_thw, &need_saved, &need_ws);
  if (saved_bytes < need_saved || ws_bytes < need_ws)
    return fail(VT_ERR_WORKSPACE, "saved (%zu < %zu) or workspace (%zu < %zu) too small", saved_bytes, need_saved,
                ws_bytes, need_ws);
  const vt_config& c = h->cfg;
  const Plan pl = make_plan(c, B, 1, gh, gw);
  const SavedLayout sl = saved_layout(c, B, gh * gw);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  auto block = [&](int i) -> char* { return static_cast<char*>(saved) + i * sl.per_layer; };
  const int K0 = 3 * c.temporal_patch * c.patch * c.patch;
  {
    ProfScope ps(CLS_UNFOLD, 0, pl.M * (4.0 * 3 * c.patch * c.patch + 2.0 * K0), st);
    cudaError_t e = launch_patch_unfold(pixels, w + pl.unfold, B, gh * c.patch, gw * c.patch, c.patch,
                                        c.temporal_patch, ORDER_BLOCK, st);
    if (e != cudaSuccess) return cuda_fail(e, "patch unfold launch");
  }
  void* x0 = c.layers > 0 ? static_cast<void*>(block(0) + sl.x) : static_cast<void*>(w + pl.x);
  if ((s = run_patch_embed(h, w + pl.unfold, x0, w, pl, st))) return s;
  for (int i = 0; i < c.layers; ++i) {
    void* out = i + 1 < c.layers ? static_cast<void*>(block(i + 1) + sl.x) : static_cast<void*>(w + pl.x);
    if ((s = run_layer_saving(h, i, block(i), sl, out, B, gh, gw, w, pl, st))) return s;
  }
  ProfScope ps(CLS_REORDER, 0, 4.0 * pl.M * c.hidden, st);
  cudaError_t e = launch_reorder_rows(w + pl.x, tower_out, B, 1, gh, gw, c.hidden, 0, st);
  if (e != cudaSuccess) return cuda_fail(e, "reorder launch");
  return VT_OK;
}

vt_status vt_backward(vt_handle* h, const void* saved, const int32_t* grid_thw, int B, const void* d_tower,
                      float* d_pixels, void* ws, size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!h->bwd_pack) return fail(VT_ERR_NOT_LOADED, "call vt_enable_backward before vt_backward");
  if (!saved || !d_tower || !d_pixels || !ws) return fail(VT_ERR_INVALID_ARG, "pointers must not be NULL");
  if (!aligned16(saved) || !aligned16(d_tower) || !aligned16(d_pixels) || !aligned16(ws))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int gh, gw;
  if ((s = check_backward_grid(h, B, grid_thw, &gh, &gw))) return s;
  size_t need_saved, need_ws;
  vt_backward_bytes(h, B, grid_thw, &need_saved, &need_ws);
  if (ws_bytes < need_ws) return fail(VT_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, need_ws);
  const vt_config& c = h->cfg;
  const int N = gh * gw, d = c.hidden;
  const BwdPlan bp = make_bwd_plan(c, B, N);
  const SavedLayout sl = saved_layout(c, B, N);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  {
    ProfScope ps(CLS_REORDER, 0, 4.0 * bp.M * d, st);
    cudaError_t e = launch_reorder_rows(d_tower, w + bp.dx, B, 1, gh, gw, d, 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "reorder launch");
  }
  for (int i = c.layers - 1; i >= 0; --i)
    if ((s = run_layer_backward(h, i, static_cast<const char*>(saved) + i * sl.per_layer, sl, B, gh, gw, w, bp, st)))
      return s;
  const int K0 = 3 * c.temporal_patch * c.patch * c.patch;
  if ((s = run_gemm(gemm_params(w + bp.dx, d, h->pe_t, d, nullptr, nullptr, 0, w + bp.hmid, K0, bp.M, K0, d,
                                ACT_NONE),
                    st)))
    return s;
  ProfScope ps(CLS_BWD_MISC, 0, 2.0 * bp.M * K0 + 4.0 * bp.M * 3 * c.patch * c.patch, st);
  cudaError_t e = launch_patch_fold(w + bp.hmid, d_pixels, B, gh * c.patch, gw * c.patch, c.patch, c.temporal_patch,
                                    ORDER_BLOCK, st);
  if (e != cudaSuccess) return cuda_fail(e, "patch fold launch");
  return VT_OK;
}

vt_status vt_tower_layer_backward_bytes(const vt_handle* h, int B, const int32_t* grid_thw, size_t* ws_bytes) {
  if (!h || !ws_bytes) return fail(VT_ERR_INVALID_ARG, "handle and output must not be NULL");
  int gh, gw;
  vt_status s = check_backward_grid(h, B, grid_thw, &gh, &gw);
  if (s) return s;
  const vt_config& c = h->cfg;
  *ws_bytes = align256(saved_layout(c, B, gh * gw).per_layer) +
              std::max(make_plan(c, B, 1, gh, gw).total, make_bwd_plan(c, B, gh * gw).total);
  return VT_OK;
}

vt_status vt_tower_layer_backward(vt_handle* h, int layer, const void* x_in, const void* dy, void* dx,
                                  const int32_t* grid_thw, int B, void* ws, size_t ws_bytes, void* stream) {
  vt_status s = check_loaded(h);
  if (s) return s;
  if (!h->bwd_pack) return fail(VT_ERR_NOT_LOADED, "call vt_enable_backward before vt_tower_layer_backward");
  if (layer < 0 || layer >= h->cfg.layers) return fail(VT_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (!x_in || !dy || !dx || !ws) return fail(VT_ERR_INVALID_ARG, "pointers must not be NULL");
  if (!aligned16(x_in) || !aligned16(dy) || !aligned16(dx) || !aligned16(ws))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int gh, gw;
  if ((s = check_backward_grid(h, B, grid_thw, &gh, &gw))) return s;
  size_t need;
  vt_tower_layer_backward_bytes(h, B, grid_thw, &need);
  if (ws_bytes < need) return fail(VT_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, need);
  const vt_config& c = h->cfg;
  const int N = gh * gw, d = c.hidden;
  const SavedLayout sl = saved_layout(c, B, N);
  const Plan pl = make_plan(c, B, 1, gh, gw);
  const BwdPlan bp = make_bwd_plan(c, B, N);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* sv = static_cast<char*>(ws);                  // the layer's saved activations
  char* w = sv + align256(sl.per_layer);              // forward, then backward scratch
  cudaError_t e;
  {  // the layer runs on 2x2-block-ordered tokens, as inside the tower
    ProfScope ps(CLS_REORDER, 0, 4.0 * pl.M * d, st);
    if ((e = launch_reorder_rows(x_in, sv + sl.x, B, 1, gh, gw, d, 1, st)) != cudaSuccess)
      return cuda_fail(e, "reorder launch");
  }
  if ((s = run_layer_saving(h, layer, sv, sl, w + pl.x, B, gh, gw, w, pl, st))) return s;
  {
    ProfScope ps(CLS_REORDER, 0, 4.0 * bp.M * d, st);
    if ((e = launch_reorder_rows(dy, w + bp.dx, B, 1, gh, gw, d, 1, st)) != cudaSuccess)
      return cuda_fail(e, "reorder launch");
  }
  if ((s = run_layer_backward(h, layer, sv, sl, B, gh, gw, w, bp, st))) return s;
  ProfScope ps(CLS_REORDER, 0, 4.0 * bp.M * d, st);
  if ((e = launch_reorder_rows(w + bp.dx, dx, B, 1, gh, gw, d, 0, st)) != cudaSuccess)
    return cuda_fail(e, "reorder launch");
  return VT_OK;
}

vt_status vt_attention_backward_workspace_bytes(int B, int H, int N, int D, size_t* out) {
  if (!out || B <= 0 || H <= 0 || N <= 0 || D <= 0) return fail(VT_ERR_INVALID_ARG, "bad arguments");
  const size_t ld = static_cast<size_t>(round8(N)), lds = (static_cast<size_t>(N) + 63) / 64 * 64;
  const size_t headT = static_cast<size_t>(B) * H * D * ld;
  const size_t tok = static_cast<size_t>(B) * N * H * D;
  *out = align256(headT * 2) + align256(tok * 2) + 2 * align256(static_cast<size_t>(B) * H * lds * 4);
  return VT_OK;
}

vt_status vt_attention_backward(const void* q, const void* k, const void* v, const void* dO, void* dqkv, int B, int H,
                                int N, int D, float scale, void* ws, size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dqkv || !ws) return fail(VT_ERR_INVALID_ARG, "pointers must not be NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dqkv) || !aligned16(ws))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (B <= 0 || H <= 0 || N <= 0) return fail(VT_ERR_INVALID_ARG, "B, H, N must be positive");
  if (!(scale > 0.f)) return fail(VT_ERR_INVALID_ARG, "scale must be positive");
  if (D != 32 && D != 80) return fail(VT_ERR_UNSUPPORTED, "the attention backward covers head_dim 32 and 80");
  if (static_cast<long long>(B) * H * N > (1ll << 31) - 256) return fail(VT_ERR_SHAPE, "too many rows");
  size_t need;
  vt_attention_backward_workspace_bytes(B, H, N, D, &need);
  if (ws_bytes < need) return fail(VT_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, need);
  const int ld = round8(N), lds = (N + 63) / 64 * 64;
  const size_t headT = static_cast<size_t>(B) * H * D * ld;
  const size_t tok = static_cast<size_t>(B) * N * H * D;
  char* w = static_cast<char*>(ws);
  void* vt_ = w;
  void* o = w + align256(headT * 2);
  float* lse = reinterpret_cast<float*>(static_cast<char*>(o) + align256(tok * 2));
  float* delta = reinterpret_cast<float*>(reinterpret_cast<char*>(lse) + align256(static_cast<size_t>(B) * H * lds * 4));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  vt_status s;
  {
    // v [B, H, N, D] -> v^T [B, H, D, ld] for the forward recomputation
    const long hnd = static_cast<long>(H) * N * D, nd = static_cast<long>(N) * D;
    const long hdl = static_cast<long>(H) * D * ld, dl = static_cast<long>(D) * ld;
    cudaError_t e = launch_transpose(v, vt_, B, H, N, D, hnd, nd, D, hdl, dl, ld, st);
    if (e != cudaSuccess) return cuda_fail(e, "transpose launch");
  }
  AttnParams a{q, k, vt_, o, B, H, N, D, ld, scale};
  a.lse = lse;
  a.ld_lse = lds;
  if ((s = run_attention(a, st))) return s;
  {
    cudaError_t e = launch_attention_delta(dO, o, delta, B, N, H, D, lds, st);
    if (e != cudaSuccess) return cuda_fail(e, "delta launch");
  }
  AttnBwdParams p{};
  p.q = q;
  p.k = k;
  p.vt = vt_;
  p.dO = dO;
  p.lse = lse;
  p.delta = delta;
  p.ld_stats = lds;
  p.dqkv = dqkv;
  p.ld_dqkv = 3 * H * D;
  p.B = B;
  p.H = H;
  p.N = N;
  p.D = D;
  p.ld = ld;
  p.scale = scale;
  return run_attention_backward(p, st);
}

vt_status vt_layernorm_backward(const void* x, const void* gamma, const void* dy, const void* dres, void* dx, int rows,
                                int cols, float eps, void* stream) {
  if (!x || !gamma || !dy || !dres || !dx) return fail(VT_ERR_INVALID_ARG, "pointers must not be NULL");
  if (rows < 0 || cols <= 0 || cols % 8) return fail(VT_ERR_INVALID_ARG, "cols must be a positive multiple of 8");
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(dy) || !aligned16(dres) || !aligned16(dx))
    return fail(VT_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return run_layernorm_backward(x, gamma, dy, dres, dx, rows, cols, eps, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
