// C ABI of libnc.so (declared in include/nc.h): configuration, workspace
// layout, argument checks and the launch sequence of the forward pass.
//
// The launch sequence follows "The Mathematics of Karpathy's nanochat",
// §High-Level Forward Pass: embedding + RMSNorm (+ smear, "nanochat depth
// sweep" card), then per block the x0 re-injection (fused into the previous
// block's last GEMM epilogue), RMSNorm, the QKV projection, RoPE + QK-norm
// (+ value embedding), windowed attention, the output projection with the
// residual add, RMSNorm, FC1 + ReLU^2, FC2 with the residual add; then backout,
// the final RMSNorm, the head with softcap and the cross-entropy.
#include <stdio.h>
#include <cmath>
#include <string.h>

#include <atomic>
#include <mutex>
#include <map>
#include <utility>

#include "nc_internal.cuh"

__device__ int g_nc_status;  // OR of 1 << NC_ERR_* bits set by kernels

namespace nc {

static thread_local int t_launches = 0;
static thread_local char t_err[256] = {0};

// optional per-launch timing (caller-owned events)
struct Timing {
  cudaEvent_t* events = nullptr;  // 2 * cap
  int* kinds = nullptr;           // cap
  int cap = 0;
  int n = 0;
  unsigned mask = 0;
  bool open = false;
};
static thread_local Timing t_timing;

void launch_begin(int kind, cudaStream_t st) {
  Timing& t = t_timing;
  t.open = false;
  if (t.events != nullptr && ((t.mask >> kind) & 1u) && t.n < t.cap) {
    cudaEventRecord(t.events[2 * t.n], st);
    t.open = true;
  }
}

void launch_end(int kind, cudaStream_t st) {
  ++t_launches;
  Timing& t = t_timing;
  if (t.open) {
    cudaEventRecord(t.events[2 * t.n + 1], st);
    t.kinds[t.n] = kind;
    ++t.n;
    t.open = false;
  }
}

static void set_err(const char* where, cudaError_t e) {
  snprintf(t_err, sizeof(t_err), "%s: %s", where, cudaGetErrorString(e));
}

void record_error(const char* where, cudaError_t e) { set_err(where, e); }

void reset_launch_count() { t_launches = 0; }

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_err(what, e);
    return NC_ERR_CUDA;
  }
  return NC_OK;
}

namespace {
std::atomic<unsigned long long> g_flag_wait_ns{kWaitLimitNs};
std::atomic<unsigned> g_flag_skew{0};
}  // namespace

void flag_wait_test(unsigned long long* limit_ns, unsigned* skew) {
  *limit_ns = g_flag_wait_ns.load();
  *skew = g_flag_skew.load();
}

namespace {
std::mutex g_optin_mu;
std::map<std::pair<const void*, int>, int> g_optin_done;  // (kernel, device) -> dynamic shared memory limit set
}  // namespace

bool smem_optin(const void* kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_err("cudaGetDevice", e);
    return false;
  }
  std::lock_guard<std::mutex> lk(g_optin_mu);
  const std::pair<const void*, int> key(kernel, dev);
  const auto it = g_optin_done.find(key);
  if (it != g_optin_done.end() && it->second >= bytes) return true;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    set_err("cudaFuncSetAttribute", e);
    return false;
  }
  g_optin_done[key] = bytes;
  return true;
}

namespace {

constexpr int kMaxDev = 64;

struct DevInfo {
  int* status = nullptr;
  int num_sms = 0;
  bool ok = false;
};
DevInfo g_dev[kMaxDev];
std::mutex g_dev_mu;

// Per-device set-up: the status word's device address and the SM count.
bool dev_info(DevInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    set_err("cudaGetDevice", e);
    return false;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.ok) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_nc_status);
    if (e != cudaSuccess) {
      set_err("cudaGetSymbolAddress", e);
      return false;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) {
      set_err("cudaDeviceGetAttribute", e);
      return false;
    }
    d.status = static_cast<int*>(p);
    d.num_sms = sms;
    d.ok = true;
  }
  *out = d;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// CTA pairs the stream-K buffers of the workspace are sized for (a device
// with more SMs than 2 * kStreamKPairs runs the GEMMs on the plain schedule)
constexpr int kStreamKPairs = 96;

struct Layout {
  size_t x, x0, xbo, xn, qkv, o, h, gate, ss, rcos, rsin, rfreq, ce_sum, ce_tgt, lse, logits, tok, tgt, loss;
  size_t skws, skflags;
  size_t total;
  int ce_tiles;
};

bool config_ok(const nc_config& c) {
  if (c.n_layer <= 0 || c.n_layer > NC_MAX_LAYERS) return false;
  if (c.n_embd <= 0 || c.n_embd % 128 != 0) return false;
  if (c.head_dim != 128 || c.n_head <= 0 || c.n_kv_head <= 0 || c.n_head % c.n_kv_head != 0) return false;
  if (c.vocab <= 0 || c.vocab_padded < c.vocab || c.vocab_padded % 64 != 0) return false;
  if (c.mlp_hidden <= 0 || c.mlp_hidden % 128 != 0) return false;
  if (c.max_T <= 0 || (c.dtype != NC_BF16 && c.dtype != NC_FP32)) return false;
  if (c.gate_channels < 0 || c.gate_channels > c.n_embd) return false;
  if (c.backout_layer >= c.n_layer) return false;
  if (!(c.softmax_scale > 0.f) || !(c.softcap > 0.f) || !(c.eps >= 0.f)) return false;
  for (int l = 0; l < c.n_layer; ++l)
    if (c.window[l] <= 0) return false;
  return true;
}

Layout layout(const nc_config& c, int max_tokens) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t M = (size_t)max_tokens;
  const size_t C = c.n_embd, D = c.head_dim;
  const size_t esz = c.dtype == NC_BF16 ? 2 : 4;
  const size_t nqkv = (size_t)(c.n_head + 2 * c.n_kv_head) * D;
  L.x = take(M * C * 4);
  L.x0 = take(M * C * 4);
  L.xbo = take(M * C * 4);
  L.xn = take(M * C * esz);
  L.qkv = take(M * nqkv * esz);
  L.o = take(M * c.n_head * D * esz);
  L.h = take(M * (size_t)c.mlp_hidden * esz);
  L.gate = take(M * c.n_kv_head * 4);
  L.ss = take(M * (C / 64) * 4);  // per-row sums of squares of the residual, per column group
  L.rcos = take((size_t)c.max_T * D / 2 * 4);
  L.rsin = take((size_t)c.max_T * D / 2 * 4);
  L.rfreq = take(D * 4);
  L.ce_tiles = 2 * ((c.vocab_padded + 127) / 128);  // per (row, 128-or-256-column tile, half)
  L.ce_sum = take(M * L.ce_tiles * 4);
  L.ce_tgt = take(M * 4);
  L.lse = take(M * 4);
  const bool simt_head = c.dtype == NC_FP32 || c.gemm_impl != 0;
  L.logits = take(simt_head ? M * (size_t)c.vocab * 4 : 0);
  // stream-K partial sums of the tcgen05 pair GEMM: one 128 x 256 fp32 tile
  // per CTA of up to kStreamKPairs CTA pairs, and one flag word per CTA
  const bool tc = c.dtype == NC_BF16 && c.gemm_impl == 0;
  L.skws = take(tc ? (size_t)kStreamKPairs * 2 * 128 * 256 * 4 : 0);
  L.skflags = take(tc ? (size_t)kStreamKPairs * 2 * 4 : 0);
  L.tok = take(M * 4);
  L.tgt = take(M * 4);
  L.loss = take(M * 4);
  L.total = off;
  return L;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

// C = A B^T with the given epilogue, on tensor cores (bf16) or CUDA cores.
bool gemm(const nc_config& c, const DevInfo& d, const void* A, int lda, const void* B, int ldb, int M,
          int N, int K, const EpiParams& ep, cudaStream_t st, const StreamK* sk = nullptr) {
  if (c.dtype == NC_BF16 && c.gemm_impl == 0)
    return launch_gemm_tc((const bf16*)A, lda, (const bf16*)B, ldb, M, N, K, ep, d.status, d.num_sms, st,
                          c.gemm_pair != 0, c.gemm_pair == 2 ? sk : nullptr);
  launch_gemm_simt(A, lda, B, ldb, M, N, K, c.dtype == NC_BF16, ep, st);
  return true;
}

EpiParams epi(int mode) {
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.mode = mode;
  return e;
}

}  // namespace

// The device status word of the current device (for launchers in other files).
bool status_word(int** out) {
  DevInfo d;
  if (!dev_info(&d)) return false;
  *out = d.status;
  return true;
}

}  // namespace nc

using namespace nc;

extern "C" {

int nc_init_config(nc_config* cfg, int depth, int max_T, int dtype, const char* window_pattern,
                   int short_window, int backout_layer) {
  if (cfg == nullptr || window_pattern == nullptr) return NC_ERR_ARG;
  if (depth <= 0 || depth > NC_MAX_LAYERS || max_T <= 0 || short_window <= 0) return NC_ERR_ARG;
  if (dtype != NC_BF16 && dtype != NC_FP32) return NC_ERR_ARG;
  const size_t plen = strlen(window_pattern);
  if (plen == 0) return NC_ERR_ARG;
  for (size_t i = 0; i < plen; ++i)
    if (window_pattern[i] != 'S' && window_pattern[i] != 'L') return NC_ERR_ARG;
  if (backout_layer >= depth) return NC_ERR_ARG;
  memset(cfg, 0, sizeof(*cfg));
  const int head_dim = 128, aspect = 64;
  cfg->n_layer = depth;
  cfg->n_embd = ((depth * aspect + head_dim - 1) / head_dim) * head_dim;
  cfg->n_head = cfg->n_embd / head_dim;
  cfg->n_kv_head = cfg->n_head;
  cfg->head_dim = head_dim;
  cfg->vocab = 32768;
  cfg->vocab_padded = ((cfg->vocab + 63) / 64) * 64;
  cfg->mlp_hidden = 4 * cfg->n_embd;
  cfg->max_T = max_T;
  cfg->dtype = dtype;
  for (int l = 0; l < depth; ++l) {
    const char ch = window_pattern[l % plen];
    cfg->window[l] = (ch == 'L' || l == depth - 1) ? max_T : short_window;
    cfg->has_ve[l] = (l % 2) == ((depth - 1) % 2);
  }
  cfg->backout_layer = backout_layer < 0 ? depth / 2 : backout_layer;
  cfg->gate_channels = 12;
  cfg->smear = 1;
  cfg->gemm_impl = 0;
  cfg->gemm_pair = 1;
  cfg->attn_impl = 0;
  cfg->qk_alpha = 1.15f;
  cfg->softmax_scale = 1.0f / sqrtf((float)head_dim);
  cfg->rope_base = 100000.0f;
  cfg->eps = 1e-6f;
  cfg->softcap = 15.0f;
  cfg->ve_gate_scale = 3.0f;
  return NC_OK;
}

size_t nc_workspace_bytes(const nc_config* cfg, int max_tokens) {
  if (cfg == nullptr || max_tokens <= 0 || !config_ok(*cfg)) return 0;
  return layout(*cfg, max_tokens).total;
}

int nc_params_init(nc_params* p, const nc_config* cfg) {
  if (p == nullptr || cfg == nullptr) return NC_ERR_ARG;
  memset(p, 0, sizeof(*p));
  p->cfg = *cfg;
  return NC_OK;
}

namespace {

// The forward pass over tokens [B, T].  With last_only, the head runs on the
// last position of each row only and writes its softcapped logits to
// out_logits [B, V] (no targets, no loss); otherwise it is the full head with
// per-token cross-entropy.
int forward_impl(const nc_params* p, const int32_t* tokens, const int32_t* targets, int B, int T,
                 float* out_loss, float* out_logits, void* stream, bool last_only) {
  t_launches = 0;
  if (p == nullptr || tokens == nullptr) return NC_ERR_ARG;
  if (last_only ? out_logits == nullptr : (targets == nullptr || out_loss == nullptr)) return NC_ERR_ARG;
  const nc_config& c = p->cfg;
  if (!config_ok(c)) return NC_ERR_SHAPE;
  if (B <= 0 || T <= 0 || T > c.max_T || (long long)B * T > (long long)p->max_tokens) return NC_ERR_SHAPE;
  if (p->wte == nullptr || p->lm_head == nullptr || p->resid_lambdas == nullptr ||
      p->x0_lambdas == nullptr || (c.smear && c.gate_channels > 0 && p->smear_gate == nullptr))
    return NC_ERR_ARG;
  for (int l = 0; l < c.n_layer; ++l) {
    const nc_layer_params& lp = p->layer[l];
    if (!lp.w_qkv || !lp.w_o || !lp.w_fc1 || !lp.w_fc2) return NC_ERR_ARG;
    if (c.has_ve[l] && (!lp.ve || !lp.ve_gate)) return NC_ERR_ARG;
    if (!aligned16(lp.w_qkv) || !aligned16(lp.w_o) || !aligned16(lp.w_fc1) || !aligned16(lp.w_fc2) ||
        (lp.ve && !aligned16(lp.ve)))
      return NC_ERR_ALIGN;
  }
  if (!aligned16(p->wte) || !aligned16(p->lm_head) || !aligned16(tokens) ||
      (!last_only && (!aligned16(targets) || !aligned16(out_loss))) || (out_logits && !aligned16(out_logits)) ||
      !aligned16(p->workspace))
    return NC_ERR_ALIGN;
  if (last_only && !last_logits_supported(c.n_embd, c.dtype == NC_BF16)) return NC_ERR_SHAPE;
  const Layout Lw = layout(c, p->max_tokens);
  if (p->workspace == nullptr || p->workspace_bytes < Lw.total) return NC_ERR_WORKSPACE;
  if (c.dtype == NC_BF16 && c.gemm_impl == 0 && c.vocab_padded % 128 != 0) return NC_ERR_SHAPE;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int M = B * T;
  const int C = c.n_embd, H = c.n_head, Hkv = c.n_kv_head, D = c.head_dim, V = c.vocab;
  const int nqkv = (H + 2 * Hkv) * D;
  const int bf = c.dtype == NC_BF16;
  void* ws = p->workspace;
  float* x = at<float>(ws, Lw.x);
  float* x0 = at<float>(ws, Lw.x0);
  float* xbo = at<float>(ws, Lw.xbo);
  void* xn = at<char>(ws, Lw.xn);
  char* qkv = at<char>(ws, Lw.qkv);
  void* o = at<char>(ws, Lw.o);
  void* h = at<char>(ws, Lw.h);
  float* gate = at<float>(ws, Lw.gate);
  float* rcos = at<float>(ws, Lw.rcos);
  float* rsin = at<float>(ws, Lw.rsin);
  float* rfreq = at<float>(ws, Lw.rfreq);
  const size_t esz = bf ? 2 : 4;

  // tensor-core path: RMSNorm is fused into the GEMMs (producers write bf16(x)
  // and per-row sums of squares, consumers scale their rows by 1 / rms)
  const bool tc = bf && c.gemm_impl == 0;
  // stream-K flags (split-tail schedule, gemm_pair == 2 only) start at 0 each
  // forward; every GEMM launch of the forward gets its own generation number.
  // Other schedules skip the memset, which would break the programmatic
  // dependent launch between the previous forward's last kernel and this one's
  // first.
  StreamK sk{nullptr, nullptr, 0u, kStreamKPairs};
  if (tc && c.gemm_pair == 2) {
    sk.ws = at<float>(ws, Lw.skws);
    sk.flags = at<unsigned>(ws, Lw.skflags);
    if (cudaMemsetAsync(sk.flags, 0, (size_t)kStreamKPairs * 2 * 4, st) != cudaSuccess) return NC_ERR_CUDA;
  }
  auto next_sk = [&]() -> const StreamK* {
    if (!tc) return nullptr;
    ++sk.gen;
    return &sk;
  };
  int tbits = 1;
  while ((1 << tbits) < T) ++tbits;
  // the tensor-core QKV epilogue computes cos / sin from the split
  // frequencies alone; the positional table serves the CUDA-core path
  launch_rope_table(rcos, rsin, tc ? 0 : T, D, c.rope_base, st, rfreq, tbits);
  float* ss = at<float>(ws, Lw.ss);
  const int ss_parts = C / (gemm_tc_bn(C) / 2);  // per-row sums of squares, one slot per epilogue warp's columns
  bf16* xb = tc ? static_cast<bf16*>(xn) : nullptr;
  launch_embed(p->wte, tokens, p->smear_gate, c.smear && c.gate_channels > 0, c.gate_channels,
               p->resid_lambdas, p->x0_lambdas, c.eps, B, T, C, V, bf, x, x0, xb, tc ? ss : nullptr,
               ss_parts, d.status, st);
  // consumer / producer settings of the fused norm
  auto norm_in = [&](EpiParams& e) {
    e.ss_in = ss;
    e.ss_in_parts = ss_parts;
    e.inv_c = 1.0f / (float)C;
    e.eps = c.eps;
  };
  auto norm_out = [&](EpiParams& e) {
    e.xb_out = xb;
    e.ldxb = C;
    e.ss_out = ss;
    e.ss_parts = ss_parts;
  };

  for (int l = 0; l < c.n_layer; ++l) {
    const nc_layer_params& lp = p->layer[l];
    const bool ve = c.has_ve[l] != 0;
    // attention sub-block
    if (!tc)
      launch_rmsnorm(x, xn, M, C, c.eps, bf, ve ? lp.ve_gate : nullptr, Hkv, c.gate_channels,
                     c.ve_gate_scale, ve ? gate : nullptr, st);
    EpiParams e = epi(tc ? EPI_QKV : EPI_STORE);
    e.out = qkv;
    e.ldo = nqkv;
    if (tc) {
      // RoPE + QK-norm, the value-embedding gate and mix run on the fp32 accumulator
      norm_in(e);
      e.T = T;
      e.qk_cols = (H + Hkv) * D;
      e.rope_fsplit = rfreq;
      e.qk_alpha = c.qk_alpha;
      e.tokens = tokens;
      e.ve = ve ? lp.ve : nullptr;
      e.gate = nullptr;
      e.gate_w = lp.ve_gate;
      e.gate_c = c.gate_channels;
      e.gate_scale = c.ve_gate_scale;
      e.x = x;
      e.ldx = C;
      e.n_kv_head = Hkv;
      e.vocab = V;
    }
    if (!gemm(c, d, xn, C, lp.w_qkv, C, M, nqkv, C, e, st, next_sk())) return NC_ERR_CUDA;
    if (!tc)
      launch_rope_qknorm_ve(qkv, nqkv, B, T, H, Hkv, D, rcos, rsin, c.qk_alpha, c.eps, tokens,
                            ve ? lp.ve : nullptr, gate, V, bf, d.status, st);
    const int w = c.window[l] >= T ? T : c.window[l];
    const char* qp = qkv;
    const char* kp = qkv + (size_t)H * D * esz;
    const char* vp = qkv + (size_t)(H + Hkv) * D * esz;
    if (bf && c.attn_impl == 0) {
      if (!launch_attn_tc((const bf16*)qp, (const bf16*)kp, (const bf16*)vp, nqkv, nqkv, nqkv, (bf16*)o, H * D,
                          B, T, H, Hkv, w, c.softmax_scale, d.status, d.num_sms, st))
        return NC_ERR_CUDA;
    } else {
      launch_attn_simt(qp, kp, vp, nqkv, nqkv, nqkv, o, H * D, B, T, H, Hkv, w, c.softmax_scale, bf, st);
    }
    e = epi(EPI_RESID);
    e.x = x;
    e.ldx = C;
    if (tc) norm_out(e);
    if (!gemm(c, d, o, H * D, lp.w_o, H * D, M, C, H * D, e, st, next_sk())) return NC_ERR_CUDA;
    // MLP sub-block
    if (!tc) launch_rmsnorm(x, xn, M, C, c.eps, bf, nullptr, 0, 0, 0.f, nullptr, st);
    e = epi(EPI_RELU2);
    e.out = h;
    e.ldo = c.mlp_hidden;
    if (tc) norm_in(e);
    if (!gemm(c, d, xn, C, lp.w_fc1, C, M, c.mlp_hidden, C, e, st, next_sk())) return NC_ERR_CUDA;
    e = epi(EPI_BLOCK_END);
    e.x = x;
    e.x0 = x0;
    e.xbo = xbo;
    e.ldx = C;
    e.capture_bo = (l == c.backout_layer);
    if (l + 1 < c.n_layer) {
      e.end_kind = 1;
      e.lam = p->resid_lambdas + l + 1;
      e.mu = p->x0_lambdas + l + 1;
    } else {
      e.end_kind = c.backout_layer >= 0 ? 2 : 0;
      e.beta = p->backout_lambda;
    }
    if (tc) norm_out(e);  // the next block's (or the head's) normalised input
    if (!gemm(c, d, h, c.mlp_hidden, lp.w_fc2, c.mlp_hidden, M, C, c.mlp_hidden, e, st, next_sk()))
      return NC_ERR_CUDA;
  }

  // final norm, head, softcap, cross-entropy
  if (last_only) {
    launch_last_logits(x, C, B, T, p->lm_head, V, C, bf, c.softcap, c.eps, out_logits, V, d.num_sms, d.status, st);
  } else if (tc) {
    const int bn = gemm_tc_bn(c.vocab_padded);
    const int tiles = 2 * ((c.vocab_padded + bn - 1) / bn);  // two epilogue halves per tile
    EpiParams e = epi(EPI_CE);
    norm_in(e);
    e.cap = c.softcap;
    e.vocab = V;
    e.logits = out_logits;
    e.ldl = V;
    e.targets = targets;
    e.ce_sum = at<float>(ws, Lw.ce_sum);
    e.ce_tgt = at<float>(ws, Lw.ce_tgt);
    e.ce_tiles = tiles;
    if (!gemm(c, d, xn, C, p->lm_head, C, M, c.vocab_padded, C, e, st)) return NC_ERR_CUDA;
    launch_ce_combine(e.ce_sum, e.ce_tgt, tiles, c.softcap, targets, M, V, out_loss, at<float>(ws, Lw.lse), d.status,
                      st);
  } else {
    launch_rmsnorm(x, xn, M, C, c.eps, bf, nullptr, 0, 0, 0.f, nullptr, st);
    float* logits = out_logits ? out_logits : at<float>(ws, Lw.logits);
    EpiParams e = epi(EPI_SOFTCAP);
    e.cap = c.softcap;
    e.vocab = V;
    e.logits = logits;
    e.ldl = V;
    launch_gemm_simt(xn, C, p->lm_head, C, M, c.vocab_padded, C, bf, e, st);
    launch_ce_rows(logits, V, targets, M, V, out_loss, d.status, st);
  }
  return check_launch(last_only ? "nc_last_logits" : "nc_forward");
}

}  // namespace

int nc_forward(const nc_params* p, const int32_t* tokens, const int32_t* targets, int B, int T,
               float* out_loss, float* out_logits, void* stream) {
  return forward_impl(p, tokens, targets, B, T, out_loss, out_logits, stream, false);
}

int nc_last_logits(const nc_params* p, const int32_t* tokens, int B, int T, float* out_logits, void* stream) {
  return forward_impl(p, tokens, nullptr, B, T, nullptr, out_logits, stream, true);
}

int nc_sample(const float* logits, int B, int V, int ldl, float temperature, int top_k, const float* uniforms,
              int32_t* out_next, void* stream) {
  t_launches = 0;
  if (logits == nullptr || uniforms == nullptr || out_next == nullptr) return NC_ERR_ARG;
  if (B <= 0 || V <= 0 || ldl < V || top_k < 0 || !(temperature >= 0.f) || !std::isfinite(temperature))
    return NC_ERR_SHAPE;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  launch_sample(logits, B, V, ldl, temperature, top_k, uniforms, out_next, d.status,
                static_cast<cudaStream_t>(stream));
  return check_launch("nc_sample");
}

int nc_generate_next(const nc_params* p, const int32_t* tokens, int B, int T, float temperature, int top_k,
                     const float* uniforms, int32_t* out_next, float* out_logits, void* stream) {
  if (uniforms == nullptr || out_next == nullptr || out_logits == nullptr) return NC_ERR_ARG;
  if (top_k < 0 || !(temperature >= 0.f) || !std::isfinite(temperature)) return NC_ERR_SHAPE;
  const int rc = forward_impl(p, tokens, nullptr, B, T, nullptr, out_logits, stream, true);
  if (rc != NC_OK) return rc;
  const int V = p->cfg.vocab;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  launch_sample(out_logits, B, V, V, temperature, top_k, uniforms, out_next, d.status,
                static_cast<cudaStream_t>(stream));
  return check_launch("nc_generate_next");
}

int nc_forward_host(const nc_params* p, const int32_t* h_tokens, const int32_t* h_targets, int B,
                    int T, float* h_out_loss, void* stream) {
  if (p == nullptr || h_tokens == nullptr || h_targets == nullptr || h_out_loss == nullptr)
    return NC_ERR_ARG;
  if (!config_ok(p->cfg)) return NC_ERR_SHAPE;
  if (B <= 0 || T <= 0 || (long long)B * T > (long long)p->max_tokens) return NC_ERR_SHAPE;
  const Layout Lw = layout(p->cfg, p->max_tokens);
  if (p->workspace == nullptr || p->workspace_bytes < Lw.total) return NC_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = (size_t)B * T;
  int32_t* dtok = at<int32_t>(p->workspace, Lw.tok);
  int32_t* dtgt = at<int32_t>(p->workspace, Lw.tgt);
  float* dloss = at<float>(p->workspace, Lw.loss);
  cudaError_t e = cudaMemcpyAsync(dtok, h_tokens, n * 4, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dtgt, h_targets, n * 4, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) {
    set_err("nc_forward_host H2D", e);
    return NC_ERR_CUDA;
  }
  const int rc = nc_forward(p, dtok, dtgt, B, T, dloss, nullptr, stream);
  if (rc != NC_OK) return rc;
  e = cudaMemcpyAsync(h_out_loss, dloss, n * 4, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) {
    set_err("nc_forward_host D2H", e);
    return NC_ERR_CUDA;
  }
  return NC_OK;
}

size_t nc_head_backward_workspace_bytes(const nc_config* cfg, int max_tokens) {
  if (cfg == nullptr || max_tokens <= 0 || !config_ok(*cfg)) return 0;
  const size_t M = (size_t)max_tokens;
  return align256(M * (size_t)cfg->vocab_padded * 2) + align256(M * (size_t)cfg->n_embd * 4) + 256;
}

int nc_head_backward(const nc_params* p, const int32_t* targets, int B, int T, float* out_dx, float* out_dw,
                     void* bwd_workspace, size_t bwd_workspace_bytes, void* stream) {
  t_launches = 0;
  if (p == nullptr || targets == nullptr || out_dx == nullptr || out_dw == nullptr) return NC_ERR_ARG;
  const nc_config& c = p->cfg;
  if (!config_ok(c)) return NC_ERR_SHAPE;
  if (c.dtype != NC_BF16 || c.gemm_impl != 0 || c.vocab_padded % 128 != 0) return NC_ERR_SHAPE;
  if (B <= 0 || T <= 0 || T > c.max_T || (long long)B * T > (long long)p->max_tokens) return NC_ERR_SHAPE;
  if (!aligned16(targets) || !aligned16(out_dx) || !aligned16(out_dw) || !aligned16(p->lm_head) ||
      !aligned16(bwd_workspace) || !aligned16(p->workspace))
    return NC_ERR_ALIGN;
  const Layout Lw = layout(c, p->max_tokens);
  if (p->workspace == nullptr || p->workspace_bytes < Lw.total) return NC_ERR_WORKSPACE;
  const size_t need = nc_head_backward_workspace_bytes(&c, p->max_tokens);
  if (bwd_workspace == nullptr || bwd_workspace_bytes < need) return NC_ERR_WORKSPACE;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int M = B * T, C = c.n_embd, V = c.vocab, Vp = c.vocab_padded;
  void* ws = p->workspace;
  char* bw = static_cast<char*>(bwd_workspace);
  bf16* dz = reinterpret_cast<bf16*>(bw);                                  // [M, Vp] bf16, rows scaled by 1/rms
  float* g = reinterpret_cast<float*>(bw + align256((size_t)p->max_tokens * Vp * 2));  // [M, C]
  float* inv_count = reinterpret_cast<float*>(bw + align256((size_t)p->max_tokens * Vp * 2) +
                                              align256((size_t)p->max_tokens * C * 4));
  const bf16* xb = at<bf16>(ws, Lw.xn);        // bf16(x) of the final residual, the head's A operand
  const float* x = at<float>(ws, Lw.x);        // the final residual (after backout), fp32
  const float* ss = at<float>(ws, Lw.ss);      // its row sums of squares, per column group
  const int ss_parts = C / (gemm_tc_bn(C) / 2);  // per-row sums of squares, one slot per epilogue warp's columns
  launch_inv_count(targets, M, inv_count, st);
  // dz' = (1/rms) dL/dz: the head GEMM recomputed, the CE gradient in its epilogue
  EpiParams e = epi(EPI_DZ);
  e.ss_in = ss;
  e.ss_in_parts = ss_parts;
  e.inv_c = 1.0f / (float)C;
  e.eps = c.eps;
  e.cap = c.softcap;
  e.vocab = V;
  e.targets = targets;
  e.lse = at<float>(ws, Lw.lse);
  e.inv_count = inv_count;
  e.out = dz;
  e.ldo = Vp;
  if (!launch_gemm_tc_layout(xb, C, 0, static_cast<const bf16*>(p->lm_head), C, 0, M, Vp, C, e, d.status, d.num_sms,
                             st))
    return NC_ERR_CUDA;
  // g = dz' W_U = (1/rms) dL/dxn; then dx = g - x r^2 (x . g) / C
  e = epi(EPI_F32);
  e.out = g;
  e.ldo = C;
  if (!launch_gemm_tc_layout(dz, Vp, 0, static_cast<const bf16*>(p->lm_head), C, 1, M, C, Vp, e, d.status, d.num_sms,
                             st))
    return NC_ERR_CUDA;
  launch_rmsnorm_bwd(x, g, out_dx, M, C, c.eps, st);
  // dW_U = dz'^T bf16(x) = dL/dz^T xn
  e = epi(EPI_F32);
  e.out = out_dw;
  e.ldo = C;
  if (!launch_gemm_tc_layout(dz, Vp, 1, xb, C, 1, V, C, M, e, d.status, d.num_sms, st)) return NC_ERR_CUDA;
  return check_launch("nc_head_backward");
}

int nc_loss_mean(const float* loss, const int32_t* targets, int n, float* out_mean, void* stream) {
  if (loss == nullptr || targets == nullptr || out_mean == nullptr || n < 0) return NC_ERR_ARG;
  launch_loss_mean(loss, targets, n, out_mean, static_cast<cudaStream_t>(stream));
  return check_launch("nc_loss_mean");
}

size_t nc_attention_workspace_bytes(int B, int T, int H, int Hkv, int D, int dtype, int rope_qknorm) {
  if (B <= 0 || T <= 0 || H <= 0 || Hkv <= 0 || D <= 0) return 0;
  if (!rope_qknorm) return 0;
  const size_t esz = dtype == NC_BF16 ? 2 : 4;
  const size_t M = (size_t)B * T;
  return align256(M * H * D * esz) + align256(M * Hkv * D * esz) + 2 * align256((size_t)T * D / 2 * 4);
}

int nc_attention(const void* q, const void* k, const void* v, void* out, int B, int T, int H,
                 int Hkv, int D, int window, int rope_qknorm, float alpha, float softmax_scale,
                 float rope_base, float eps, int dtype, void* workspace, size_t workspace_bytes,
                 void* stream) {
  t_launches = 0;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return NC_ERR_ARG;
  if (dtype != NC_BF16 && dtype != NC_FP32) return NC_ERR_ARG;
  if (!(softmax_scale > 0.f) || !(eps >= 0.f)) return NC_ERR_ARG;
  if (B <= 0 || T <= 0 || H <= 0 || Hkv <= 0) return NC_ERR_SHAPE;
  if (D != 128 || Hkv <= 0 || H % Hkv != 0) return NC_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return NC_ERR_ALIGN;
  const size_t need = nc_attention_workspace_bytes(B, T, H, Hkv, D, dtype, rope_qknorm);
  if (rope_qknorm && (workspace == nullptr || workspace_bytes < need)) return NC_ERR_WORKSPACE;
  if (rope_qknorm && !aligned16(workspace)) return NC_ERR_ALIGN;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bf = dtype == NC_BF16;
  const size_t esz = bf ? 2 : 4;
  const size_t M = (size_t)B * T;
  const int w = (window <= 0 || window >= T) ? T : window;
  const void* qa = q;
  const void* ka = k;
  if (rope_qknorm) {
    char* base = static_cast<char*>(workspace);
    void* qo = base;
    void* ko = base + align256(M * H * D * esz);
    float* rc = reinterpret_cast<float*>(base + align256(M * H * D * esz) + align256(M * Hkv * D * esz));
    float* rs = rc + align256((size_t)T * D / 2 * 4) / 4;
    launch_rope_table(rc, rs, T, D, rope_base, st);
    launch_rope_qknorm_copy(q, k, qo, ko, B, T, H, Hkv, D, rc, rs, alpha, eps, bf, st);
    qa = qo;
    ka = ko;
  }
  if (bf) {
    if (!launch_attn_tc((const bf16*)qa, (const bf16*)ka, (const bf16*)v, H * D, Hkv * D, Hkv * D, (bf16*)out,
                        H * D, B, T, H, Hkv, w, softmax_scale, d.status, d.num_sms, st))
      return NC_ERR_CUDA;
  } else {
    launch_attn_simt(qa, ka, v, H * D, Hkv * D, Hkv * D, out, H * D, B, T, H, Hkv, w, softmax_scale, bf, st);
  }
  return check_launch("nc_attention");
}

size_t nc_routing_attention_workspace_bytes(int B, int T, int H, int D) {
  if (B <= 0 || T <= 0 || H <= 0 || D <= 0) return 0;
  return align256((size_t)B * T * H * D * 2);
}

int nc_routing_attention(const void* q2, const void* k2, const void* v2, const void* q1, const void* k1, void* out,
                         int B, int T, int H, int Hkv, int D, int window, float gate_logit, float softmax_scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
  t_launches = 0;
  if (!q2 || !k2 || !v2 || !q1 || !k1 || !out) return NC_ERR_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(gate_logit)) return NC_ERR_ARG;
  if (B <= 0 || T <= 0 || H <= 0 || Hkv <= 0 || D != 128 || H % Hkv != 0) return NC_ERR_SHAPE;
  if (!aligned16(q2) || !aligned16(k2) || !aligned16(v2) || !aligned16(q1) || !aligned16(k1) || !aligned16(out) ||
      !aligned16(workspace))
    return NC_ERR_ALIGN;
  if (workspace == nullptr || workspace_bytes < nc_routing_attention_workspace_bytes(B, T, H, D))
    return NC_ERR_WORKSPACE;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // g = softplus(gate_logit), evaluated without overflow
  const double a = gate_logit;
  const float g = (float)(a > 0 ? a + log1p(exp(-a)) : log1p(exp(a)));
  bf16* q1s = static_cast<bf16*>(workspace);
  launch_scale_bf16(static_cast<const bf16*>(q1), q1s, (long long)B * T * H * D, g, d.num_sms, st);
  const int w = (window <= 0 || window >= T) ? T : window;
  if (!launch_attn_route_tc(static_cast<const bf16*>(q2), static_cast<const bf16*>(k2), static_cast<const bf16*>(v2),
                            q1s, static_cast<const bf16*>(k1), static_cast<bf16*>(out), B, T, H, Hkv, w,
                            softmax_scale, d.status, d.num_sms, st))
    return check_launch("nc_routing_attention") == NC_OK ? NC_ERR_CUDA : NC_ERR_CUDA;
  return check_launch("nc_routing_attention");
}

}  // extern "C"

namespace {

// Nested block widths -> cumulative ends; false unless 1 <= k <= 8, every
// width a positive multiple of 64 and their sum C.
bool prefix_blocks(const int* widths, int k, int C, PrefixBlocks* pb) {
  if (widths == nullptr || k < 1 || k > kMaxPrefixBlocks) return false;
  memset(pb, 0, sizeof(*pb));
  pb->k = k;
  int e = 0;
  for (int a = 0; a < k; ++a) {
    if (widths[a] <= 0 || widths[a] % 64 != 0) return false;
    e += widths[a];
    pb->end[a] = e;
  }
  return e == C;
}

}  // namespace

extern "C" {

int nc_prefix_rmsnorm(const float* x, int M, int C, const int* widths, int k, float eps, void* out, int out_bf16,
                      void* stream) {
  t_launches = 0;
  if (x == nullptr || out == nullptr || !(eps >= 0.f)) return NC_ERR_ARG;
  PrefixBlocks pb;
  if (M < 0 || C <= 0 || !prefix_blocks(widths, k, C, &pb)) return NC_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(out)) return NC_ERR_ALIGN;
  if (M == 0) return NC_OK;
  launch_prefix_rmsnorm(x, M, C, pb, eps, out, out_bf16, static_cast<cudaStream_t>(stream));
  return check_launch("nc_prefix_rmsnorm");
}

int nc_btl_linear(const void* x, const void* w, float* y, int M, int C_in, int C_out, const int* in_widths,
                  const int* out_widths, int k, void* stream) {
  t_launches = 0;
  if (x == nullptr || w == nullptr || y == nullptr) return NC_ERR_ARG;
  GemmKLimit kl;
  if (M < 0 || C_in <= 0 || C_out <= 0 || C_out % 256 != 0 || !prefix_blocks(in_widths, k, C_in, &kl.in) ||
      !prefix_blocks(out_widths, k, C_out, &kl.out))
    return NC_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return NC_ERR_ALIGN;
  if (M == 0) return NC_OK;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.mode = EPI_F32;
  e.out = y;
  e.ldo = C_out;
  if (!launch_gemm_tc(static_cast<const bf16*>(x), C_in, static_cast<const bf16*>(w), C_in, M, C_out, C_in, e,
                      d.status, d.num_sms, static_cast<cudaStream_t>(stream), true, nullptr, &kl))
    return NC_ERR_CUDA;
  return check_launch("nc_btl_linear");
}

size_t nc_prefix_ce_workspace_bytes(int M, int C, int V_pad) {
  if (M <= 0 || C <= 0 || V_pad <= 0) return 0;
  const size_t tiles = 2 * ((size_t)V_pad / 128);
  return align256((size_t)M * C * 2) + align256((size_t)M * tiles * 4) + 2 * align256((size_t)M * 4);
}

int nc_prefix_ce(const float* x, const void* w_u, const int32_t* targets, float* out_loss, int M, int C, int V,
                 int V_pad, const int* widths, int k, float eps, float cap, void* workspace, size_t workspace_bytes,
                 void* stream) {
  t_launches = 0;
  if (x == nullptr || w_u == nullptr || targets == nullptr || out_loss == nullptr) return NC_ERR_ARG;
  if (!(eps >= 0.f) || !(cap > 0.f)) return NC_ERR_ARG;
  PrefixBlocks pb;
  if (M <= 0 || C <= 0 || V <= 0 || V_pad < V || V_pad % 256 != 0 || !prefix_blocks(widths, k, C, &pb))
    return NC_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w_u) || !aligned16(targets) || !aligned16(out_loss) || !aligned16(workspace))
    return NC_ERR_ALIGN;
  if (workspace == nullptr || workspace_bytes < nc_prefix_ce_workspace_bytes(M, C, V_pad)) return NC_ERR_WORKSPACE;
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  bf16* xn = reinterpret_cast<bf16*>(ws);
  const int tiles = 2 * (V_pad / 256);  // partial sums per row: (256-column pair tile, column half)
  float* ce_sum = reinterpret_cast<float*>(ws + align256((size_t)M * C * 2));
  float* ce_tgt = reinterpret_cast<float*>(ws + align256((size_t)M * C * 2) + align256((size_t)M * (2 * (V_pad / 128)) * 4));
  float* lse = ce_tgt + align256((size_t)M * 4) / 4;
  // the normalised prefix of every submodel at once (block a scaled by the
  // RMS of the prefix up to it), bf16 as the head GEMM's A operand
  launch_prefix_rmsnorm(x, M, C, pb, eps, xn, 1, st);
  for (int j = 0; j < k; ++j) {
    // submodel j + 1: the first C_j columns of x_n and of W_U
    EpiParams e;
    memset(&e, 0, sizeof(e));
    e.mode = EPI_CE;
    e.cap = cap;
    e.vocab = V;
    e.targets = targets;
    e.ce_sum = ce_sum;
    e.ce_tgt = ce_tgt;
    e.ce_tiles = tiles;
    if (!launch_gemm_tc(xn, C, static_cast<const bf16*>(w_u), C, M, V_pad, pb.end[j], e, d.status, d.num_sms, st, true))
      return NC_ERR_CUDA;
    launch_ce_combine(ce_sum, ce_tgt, tiles, cap, targets, M, V, out_loss + (size_t)j * M, lse, d.status, st);
  }
  return check_launch("nc_prefix_ce");
}

int nc_get_status(void* stream, int* out_bits) {
  DevInfo d;
  if (!dev_info(&d)) return NC_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  int bits = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&bits, d.status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(d.status, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    set_err("nc_get_status", e);
    return NC_ERR_CUDA;
  }
  if (out_bits) *out_bits = bits;
  if (bits & kStatusTimeout) return NC_ERR_TIMEOUT;
  if (bits & kStatusData) return NC_ERR_DATA;
  return NC_OK;
}

const char* nc_status_string(int s) {
  switch (s) {
    case NC_OK: return "ok";
    case NC_ERR_ARG: return "invalid argument";
    case NC_ERR_SHAPE: return "unsupported or inconsistent shape";
    case NC_ERR_ALIGN: return "pointer not 16-byte aligned";
    case NC_ERR_CUDA: return "CUDA runtime error";
    case NC_ERR_DATA: return "token or target id out of range (clamped on the device)";
    case NC_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case NC_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

const char* nc_last_error(void) { return t_err; }

int nc_last_launch_count(void) { return t_launches; }

int nc_set_flag_wait_test(int skew, double wait_limit_ms) {
  if (skew < 0 || !(wait_limit_ms > 0.0) || wait_limit_ms > 1000.0) return NC_ERR_ARG;
  g_flag_wait_ns.store((unsigned long long)(wait_limit_ms * 1e6));
  g_flag_skew.store((unsigned)skew);
  return NC_OK;
}

int nc_set_launch_timing(void** events, int* kinds, int capacity, unsigned kind_mask) {
  if (events != nullptr && (kinds == nullptr || capacity <= 0)) return NC_ERR_ARG;
  t_timing = Timing();
  t_timing.events = reinterpret_cast<cudaEvent_t*>(events);
  t_timing.kinds = kinds;
  t_timing.cap = events ? capacity : 0;
  t_timing.mask = kind_mask;
  return NC_OK;
}

int nc_launch_timing_count(void) { return t_timing.n; }

const char* nc_kernel_name(int kind) {
  static const char* names[KK_COUNT] = {
      "embed_norm_smear", "rmsnorm", "rope_table", "rope_qknorm", "gemm_tcgen05", "gemm_cuda_core",
      "attention_tcgen05", "attention_cuda_core", "ce_combine", "ce_rows", "loss_mean", "last_logits",
      "sample", "gemm_tcgen05_bwd", "head_bwd_rows", "prefix_rmsnorm"};
  return (kind >= 0 && kind < KK_COUNT) ? names[kind] : "unknown";
}

size_t nc_sizeof(int which) {
  switch (which) {
    case 0: return sizeof(nc_config);
    case 1: return sizeof(nc_layer_params);
    case 2: return sizeof(nc_params);
    default: return 0;
  }
}

}  // extern "C"
