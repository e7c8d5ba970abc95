// Internal declarations shared by the CUDA translation units of libnc.so.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nc.h"

namespace nc {

// bits of the device status word
constexpr int kStatusData = 1 << NC_ERR_DATA;
constexpr int kStatusTimeout = 1 << NC_ERR_TIMEOUT;

// one second: upper bound of any wait inside a kernel
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

using bf16 = __nv_bfloat16;

template <typename T> struct Act;
template <> struct Act<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
  static __device__ __forceinline__ float from(float v) { return v; }
};
template <> struct Act<bf16> {
  static __device__ __forceinline__ float ld(const bf16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(bf16* p, float v) { *p = __float2bfloat16_rn(v); }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

// ---------------------------------------------------------------------------
// Epilogue description shared by the GEMM kernels (CUDA-core and tcgen05).
// C = A B^T is computed in fp32; the epilogue decides what happens to it.
// ---------------------------------------------------------------------------
enum EpiMode : int {
  EPI_STORE = 0,     // out[m, n] = acc                       (act dtype)
  EPI_RELU2 = 1,     // out[m, n] = max(acc, 0)^2             (act dtype)
  EPI_RESID = 2,     // x[m, n] += acc                        (fp32 residual)
  EPI_BLOCK_END = 3, // x += acc; capture x_bo; then re-inject for the next block or apply backout
  EPI_SOFTCAP = 4,   // logits[m, n] = cap tanh(acc / cap)    (fp32; CUDA-core path)
  EPI_CE = 5,        // softcap + per-(row, tile) log-sum-exp partials (+ optional logits)
  EPI_QKV = 6,       // q, k heads: RoPE + QK-norm; v heads: + gate * VE[tok]; bf16 out (tcgen05 path)
  EPI_DZ = 7,        // head backward: d loss / d z of the softcapped CE, times 1/rms of the row, bf16 out
  EPI_F32 = 8        // out[m, n] = acc (fp32)
};

struct EpiParams {
  int mode;
  void* out;          // EPI_STORE / EPI_RELU2: act [M, ldo]
  int ldo;
  float* x;           // residual [M, ldx] fp32
  const float* x0;    // [M, ldx]
  float* xbo;         // [M, ldx]
  int ldx;
  int capture_bo;     // EPI_BLOCK_END: store x_bo = x + acc
  int end_kind;       // EPI_BLOCK_END: 0 = nothing after, 1 = x = lam x + mu x0, 2 = x -= beta x_bo
  const float* lam;   // device scalars of the next block: lambda_{l+1}, mu_{l+1}
  const float* mu;
  float beta;
  // EPI_SOFTCAP / EPI_CE
  float cap;
  int vocab;          // columns >= vocab are padding: not written, not in the LSE
  float* logits;      // [M, ldl] fp32 or NULL
  int ldl;
  const int32_t* targets;  // [M]
  float* ce_sum;      // [M, n_tiles]: sum over the tile's columns of exp(zhat - cap)
  float* ce_tgt;      // [M]
  int ce_tiles;
  // EPI_QKV (out/ldo as for EPI_STORE)
  int T;              // positions per row (position = m % T)
  int qk_cols;        // (H + H_kv) * D: columns below this are q and k heads
  const float* rope_fsplit;  // [2, D/2]: per-frequency cycles per position, split hi | lo (see k_rope_table)
  float qk_alpha, eps;
  const int32_t* tokens;  // [M]
  const void* ve;     // [V, H_kv D] or NULL
  const float* gate;  // [M, H_kv] precomputed gates (CUDA-core path), or NULL
  int n_kv_head;
  // RMSNorm fused into the tcgen05 GEMMs ("The Mathematics of Karpathy's
  // nanochat", §RMS Normalization): RMSNorm(x) W^T = (bf16(x) W^T) / rms(x).
  // Producer side (EPI_RESID / EPI_BLOCK_END): besides the fp32 x also write
  // xb = bf16(x) and, per row, the sum of squares of the new x over each
  // BN/2-column group: ss_out[m, n / (BN/2)].
  bf16* xb_out;
  int ldxb;
  float* ss_out;
  int ss_parts;       // groups per row (C / (BN/2))
  // Consumer side (EPI_QKV / EPI_RELU2 / EPI_CE, A operand = xb): each row is
  // scaled by 1 / sqrt(sum_j ss_in[m, j] / C + eps) before the epilogue op.
  const float* ss_in;
  int ss_in_parts;
  float inv_c;        // 1 / C
  // EPI_DZ (A = bf16(x), rows scaled by 1 / rms through ss_in as for EPI_CE;
  // targets, vocab and cap as for EPI_CE): with zhat = cap tanh(z / cap),
  //   out[m, n] = bf16( rscale_m * inv_count * (exp(zhat - lse[m]) - [n == y_m]) * (1 - (zhat / cap)^2) )
  // for rows with a valid target and n < vocab, 0 elsewhere
  const float* lse;        // [M] log-sum-exp of the row's softcapped logits
  const float* inv_count;  // device scalar: 1 / (number of valid targets), 0 if none
  // value-embedding gate inside the QKV epilogue (when gate == NULL):
  // g = gate_scale * sigmoid(rstd * x[m, :gate_c] . gate_w[h, :gate_c])
  const float* gate_w;
  int gate_c;
  float gate_scale;
};

// launchers (host functions), all asynchronous on `st`
void launch_embed(const void* wte, const int32_t* tokens, const float* smear_gate, int smear,
                  int gate_channels, const float* lam0, const float* mu0, float eps, int B, int T, int C, int V,
                  int act_bf16, float* x, float* x0, bf16* xb, float* ss, int ss_parts, int* status,
                  cudaStream_t st);
void launch_rmsnorm(const float* x, void* xn, int M, int C, float eps, int act_bf16,
                    const float* ve_gate, int Hkv, int gate_channels, float gate_scale, float* gate_out,
                    cudaStream_t st);
void launch_rope_table(float* cos_t, float* sin_t, int T, int D, float base, cudaStream_t st,
                       float* fsplit = nullptr, int tbits = 0);
void launch_rope_qknorm_ve(void* qkv, int ld, int B, int T, int H, int Hkv, int D,
                           const float* cos_t, const float* sin_t, float alpha, float eps,
                           const int32_t* tokens, const void* ve, const float* gate, int V,
                           int act_bf16, int* status, cudaStream_t st);
void launch_rope_qknorm_copy(const void* q, const void* k, void* qo, void* ko, int B, int T, int H,
                             int Hkv, int D, const float* cos_t, const float* sin_t, float alpha,
                             float eps, int act_bf16, cudaStream_t st);
void launch_ce_rows(const float* logits, int ldl, const int32_t* targets, int M, int V, float* loss,
                    int* status, cudaStream_t st);
void launch_ce_combine(const float* ce_sum, const float* ce_tgt, int n_tiles, float offset,
                       const int32_t* targets, int M, int V, float* loss, float* lse, int* status,
                       cudaStream_t st);
// head backward helpers: 1 / (number of targets != -1) into *inv_count, and
// the RMSNorm backward dx = g - x r^2 (x . g) / C with r = 1 / rms(x) per row
// (g = r * dL/dxn, fp32 [M, C])
void launch_inv_count(const int32_t* targets, int n, float* inv_count, cudaStream_t st);
// out = bf16(g * in), n a multiple of 8 elements, 16-byte aligned buffers
void launch_scale_bf16(const bf16* in, bf16* out, long long n, float g, int num_sms, cudaStream_t st);
void launch_rmsnorm_bwd(const float* x, const float* g, float* dx, int M, int C, float eps, cudaStream_t st);
// Nested blocks of a width: block a is [end[a-1], end[a]) (end[-1] = 0).
constexpr int kMaxPrefixBlocks = 8;
struct PrefixBlocks {
  int k;
  int end[kMaxPrefixBlocks];
};
// PrefixRMSNorm of x [M, C] fp32 into out (bf16 when out_bf16, else fp32).
void launch_prefix_rmsnorm(const float* x, int M, int C, const PrefixBlocks& pb, float eps, void* out, int out_bf16,
                           cudaStream_t st);
void launch_loss_mean(const float* loss, const int32_t* targets, int n, float* out, cudaStream_t st);
// generation: softcapped logits of the last position of each of B rows
// (x: the final fp32 residual [B T, ldx]; W: lm_head [V_padded, C], bf16 or
// fp32), and one token per row drawn from logits [B, ldl]
void launch_last_logits(const float* x, int ldx, int B, int T, const void* W, int V, int C, bool bf, float cap,
                        float eps, float* out, int ldo, int num_sms, int* status, cudaStream_t st);
bool last_logits_supported(int C, bool bf);  // C <= 2304 (bf16) / 1280 (fp32)
void launch_sample(const float* logits, int B, int V, int ldl, float temperature, int top_k,
                   const float* uniforms, int32_t* out, int* status, cudaStream_t st);

// CUDA-core GEMM: C[M, N] = A[M, K] B[N, K]^T, fp32 accumulate
void launch_gemm_simt(const void* A, int lda, const void* Bm, int ldb, int M, int N, int K,
                      int act_bf16, const EpiParams& ep, cudaStream_t st);
// CUDA-core attention over q/k/v with row strides (in elements)
void launch_attn_simt(const void* q, const void* k, const void* v, int ldq, int ldk, int ldv,
                      void* o, int ldo, int B, int T, int H, int Hkv, int window, float scale,
                      int act_bf16, cudaStream_t st);

// tcgen05 GEMM (bf16 only).  Returns false if the tensor maps cannot be built.
int gemm_tc_bn(int N);  // output tile width the tcgen05 GEMM uses for N columns
// pair = true selects the CTA-pair (cta_group::2) kernel when N % 256 == 0.
// With sk given, the pair kernel may use a stream-K schedule: ws holds
// 2 * max_pairs partial tiles of 128 x 256 floats, flags 2 * max_pairs words
// that start below gen (gen must differ between launches that share them).
struct StreamK {
  float* ws;
  unsigned* flags;
  unsigned gen;
  int max_pairs;
};
// Block lower triangular B (pair kernel): output columns below out.end[a]
// read only K elements below in.end[a] (the rest of B must be zero there).
struct GemmKLimit {
  PrefixBlocks out, in;
};
bool launch_gemm_tc(const bf16* A, int lda, const bf16* Bm, int ldb, int M, int N, int K,
                    const EpiParams& ep, int* status, int num_sms, cudaStream_t st, bool pair,
                    const StreamK* sk = nullptr, const GemmKLimit* kl = nullptr);
// tcgen05 GEMM with operands in either layout, single-CTA kernel (bf16):
// C[M, N] = A[M, K] B[N, K]^T where A is stored row-major [M, lda] when
// a_mn == 0 (K contiguous) or as its transpose [K, lda] when a_mn == 1 (M
// contiguous), likewise B ([N, ldb] or [K, ldb]).  K need not be a multiple
// of 64 (out-of-range k reads zeros).  Used by the head backward.
bool launch_gemm_tc_layout(const bf16* A, int lda, int a_mn, const bf16* Bm, int ldb, int b_mn, int M, int N,
                           int K, const EpiParams& ep, int* status, int num_sms, cudaStream_t st);
// tcgen05 attention (bf16 only)
// pass-2 routing attention: logits scale (q2 . k2 + q1s . k1) with q1s = g q1
// already scaled; all inputs [B, T, heads, 128] contiguous, o [B, T, H, 128]
bool launch_attn_route_tc(const bf16* q2, const bf16* k2, const bf16* v2, const bf16* q1s, const bf16* k1, bf16* o,
                          int B, int T, int H, int Hkv, int window, float scale, int* status, int num_sms,
                          cudaStream_t st);
bool launch_attn_tc(const bf16* q, const bf16* k, const bf16* v, int ldq, int ldk, int ldv, bf16* o,
                    int ldo, int B, int T, int H, int Hkv, int window, float scale, int* status,
                    int num_sms, cudaStream_t st);

// Raise `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device.  The attribute belongs to the device's context, so it is set per
// (kernel, device): a process that drives several devices sets it on each,
// and a later request for more bytes than the last one raises it again.  Returns false, with the CUDA error recorded for nc_last_error(),
// when the device cannot be queried or the attribute cannot be set.
bool smem_optin(const void* kernel, int bytes);
template <typename... KArgs>
bool smem_optin(void (*kernel)(KArgs...), int bytes) {
  return smem_optin(reinterpret_cast<const void*>(kernel), bytes);
}
// Settings of nc_set_flag_wait_test(): the limit (ns) of the split-K
// partial-sum flag wait and the generation offset that wait expects (0 in
// normal operation; non-zero makes the flags it waits for never arrive).
void flag_wait_test(unsigned long long* limit_ns, unsigned* skew);
// Record a CUDA error for nc_last_error() (this host thread).
void record_error(const char* where, cudaError_t e);
// Start a new launch count for nc_last_launch_count() (this host thread).
void reset_launch_count();
// NC_OK, or NC_ERR_CUDA with the error recorded, after the launches of an
// entry point (cudaGetLastError).
int check_launch(const char* what);

// Kernel kinds, for the launch counter and the optional per-launch timing.
enum KernelKind : int {
  KK_EMBED = 0, KK_RMSNORM, KK_ROPE_TABLE, KK_ROPE_QKNORM, KK_GEMM_TC, KK_GEMM_SIMT, KK_ATTN_TC,
  KK_ATTN_SIMT, KK_CE_COMBINE, KK_CE_ROWS, KK_LOSS_MEAN, KK_LAST_LOGITS, KK_SAMPLE, KK_GEMM_TC_BWD,
  KK_HEAD_BWD_ROWS, KK_PREFIX_NORM, KK_COUNT
};
// Every launcher holds one of these around its kernel launch: it counts the
// launch (per host thread) and, when the caller enabled timing for this kind,
// records a CUDA event before and after the launch on `st`.
void launch_begin(int kind, cudaStream_t st);
void launch_end(int kind, cudaStream_t st);
struct LaunchScope {
  int kind;
  cudaStream_t st;
  LaunchScope(int k, cudaStream_t s) : kind(k), st(s) { launch_begin(k, s); }
  ~LaunchScope() { launch_end(kind, st); }
};

// Programmatic dependent launch.  Kernels launched through launch_pdl may be
// scheduled while the previous kernel on the stream is still finishing, so
// each of them runs pdl_launch_dependents() first (letting the next kernel be
// scheduled in turn) and pdl_wait() before its first access to global memory:
// pdl_wait() returns once the previous kernel has completed and its writes
// are visible (at once when there is no such kernel).  Only set-up work that
// touches no global memory (barrier init, TMEM allocation, descriptor
// prefetch) runs before it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace nc
