// Row-wise, HBM-bound kernels of the forward pass: token embedding + RMSNorm +
// smear, pre-norm RMSNorm (+ value-embedding gate), RoPE + QK-norm (+ value
// embedding mix), cross-entropy reductions.
//
// Equations: "The Mathematics of Karpathy's nanochat", §RMS Normalization,
// §Rotary Position Embeddings, §Value Embeddings (ResFormer), §QK-Norm with
// Sharpening, §Logit Softcap, §Cross-Entropy Loss; smear after the embedding
// norm per the "nanochat depth sweep" card (Architecture list) and "Reading
// nanochat Source" §5.1.
#include "nc_internal.cuh"

namespace nc {

namespace {

template <typename T>
__device__ __forceinline__ float ldf(const T* p) { return Act<T>::ld(p); }

__device__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < nw; ++i) s += red[i];  // same order in every thread
  return s;
}

// x_hat_t = RMSNorm(W_E[tok_t]); x_t = x_hat_t + s_t x_hat_{t-1} (t >= 1) with
// s_t = sigmoid(w_sm . x_hat_t[:gc]); x0 = x; then the first block's
// re-injection x = lam0 x + mu0 x0.  One CTA per token.
template <typename T>
__global__ void k_embed(const T* __restrict__ wte, const int32_t* __restrict__ tokens,
                        const float* __restrict__ smear_gate, int smear, int gc,
                        const float* __restrict__ lam0p, const float* __restrict__ mu0p, float eps, int T_, int C, int V, float* __restrict__ x, float* __restrict__ x0,
                        bf16* __restrict__ xb, float* __restrict__ ss, int ss_parts, int* status) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ float sh[];  // [2C] rows + [32] reduction
  float* cur = sh;
  float* prev = sh + C;
  float* red = sh + 2 * C;
  const int m = blockIdx.x;
  const int t = m % T_;
  int tok = tokens[m];
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) atomicOr(status, kStatusData);
    tok = min(max(tok, 0), V - 1);
  }
  const bool has_prev = smear && t > 0;
  int tokp = has_prev ? tokens[m - 1] : 0;
  tokp = min(max(tokp, 0), V - 1);
  float s1 = 0.f, s2 = 0.f;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const float e = ldf(wte + (size_t)tok * C + c);
    cur[c] = e;
    s1 += e * e;
    if (has_prev) {
      const float ep = ldf(wte + (size_t)tokp * C + c);
      prev[c] = ep;
      s2 += ep * ep;
    }
  }
  s1 = block_sum(s1, red);
  s2 = block_sum(s2, red);
  const float r1 = 1.0f / sqrtf(s1 / (float)C + eps);
  const float r2 = has_prev ? 1.0f / sqrtf(s2 / (float)C + eps) : 0.f;
  float g = 0.f;
  if (has_prev) {
    float d = 0.f;
    for (int c = threadIdx.x; c < gc; c += blockDim.x) d += smear_gate[c] * (cur[c] * r1);
    d = block_sum(d, red);
    g = sigmoidf_(d);
  }
  const float lam0 = *lam0p, mu0 = *mu0p;
  float s3 = 0.f;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float xh = cur[c] * r1;
    if (has_prev) xh += g * (prev[c] * r2);
    x0[(size_t)m * C + c] = xh;
    const float v = lam0 * xh + mu0 * xh;
    x[(size_t)m * C + c] = v;
    if (xb != nullptr) {
      xb[(size_t)m * C + c] = __float2bfloat16_rn(v);
      s3 += v * v;
    }
  }
  if (xb != nullptr) {
    // the first block's norm input: sum of squares in slot 0, other slots 0
    s3 = block_sum(s3, red);
    for (int j = threadIdx.x; j < ss_parts; j += blockDim.x) ss[(size_t)m * ss_parts + j] = j == 0 ? s3 : 0.f;
  }
}

// xn = RMSNorm(x) (act dtype), one warp per row; optionally the value-embedding
// gate g[m, h] = gate_scale * sigmoid(xn[:gc] . W_gate[h]) from the fp32
// normalised values.
template <typename T>
__global__ void k_rmsnorm(const float* __restrict__ x, T* __restrict__ xn, int M, int C, float eps,
                          const float* __restrict__ wg, int Hkv, int gc, float gscale,
                          float* __restrict__ gout) {
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)m * C);
  const int n4 = C >> 2;
  float ss = 0.f;
  for (int i = lane; i < n4; i += 32) {
    const float4 v = xr[i];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)C + eps);
  T* out = xn + (size_t)m * C;
  for (int i = lane; i < n4; i += 32) {
    const float4 v = xr[i];
    Act<T>::st(out + 4 * i + 0, v.x * r);
    Act<T>::st(out + 4 * i + 1, v.y * r);
    Act<T>::st(out + 4 * i + 2, v.z * r);
    Act<T>::st(out + 4 * i + 3, v.w * r);
  }
  if (gout != nullptr) {
    const float* xrow = x + (size_t)m * C;
    for (int h = lane; h < Hkv; h += 32) {
      float d = 0.f;
      for (int c = 0; c < gc; ++c) d += wg[h * gc + c] * (xrow[c] * r);
      gout[(size_t)m * Hkv + h] = gscale * sigmoidf_(d);
    }
  }
}

template <>
__global__ void k_rmsnorm<bf16>(const float* __restrict__ x, bf16* __restrict__ xn, int M, int C,
                                float eps, const float* __restrict__ wg, int Hkv, int gc,
                                float gscale, float* __restrict__ gout) {
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)m * C);
  const int n4 = C >> 2;
  float ss = 0.f;
  for (int i = lane; i < n4; i += 32) {
    const float4 v = xr[i];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)C + eps);
  uint2* out = reinterpret_cast<uint2*>(xn + (size_t)m * C);
  for (int i = lane; i < n4; i += 32) {
    const float4 v = xr[i];
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x * r, v.y * r);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z * r, v.w * r);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    out[i] = u;
  }
  if (gout != nullptr) {
    const float* xrow = x + (size_t)m * C;
    for (int h = lane; h < Hkv; h += 32) {
      float d = 0.f;
      for (int c = 0; c < gc; ++c) d += wg[h * gc + c] * (xrow[c] * r);
      gout[(size_t)m * Hkv + h] = gscale * sigmoidf_(d);
    }
  }
}

// cos/sin of phi_{t,j} = t * base^(-2j/D), evaluated in double and rounded
// once to fp32 (an fp32 product t * omega would lose ~5e-4 rad at t ~ 8k).
// Also, when fsplit is given, the rotation frequencies in cycles per
// position, f_j = omega_j / (2 pi), split as fh_j + fl_j: fh_j keeps
// 24 - tbits significant bits, so that t * fh_j is exact in fp32 for every
// t < 2^tbits, and fl_j is the rest (fsplit = fh[0..D/2) | fl[0..D/2)).  The
// phase t f_j mod 1 then follows in fp32 to about 1e-7 cycles.
__global__ void k_rope_table(float* cos_t, float* sin_t, int T_, int D, double base, float* fsplit, int tbits) {
  pdl_launch_dependents();
  pdl_wait();
  const int half = D / 2;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (fsplit != nullptr && i < half) {
    const double f = pow(base, -2.0 * (double)i / (double)D) / (2.0 * 3.14159265358979323846);
    int e = 0;
    frexp(f, &e);  // f = m 2^e, m in [0.5, 1)
    const int keep = 24 - tbits;
    const double fh = ldexp(rint(ldexp(f, keep - e)), e - keep);
    fsplit[i] = (float)fh;
    fsplit[half + i] = (float)(f - fh);
  }
  if (i >= T_ * half) return;
  const int t = i / half, j = i % half;
  const double omega = pow(base, -2.0 * (double)j / (double)D);
  double s, c;
  sincos((double)t * omega, &s, &c);
  cos_t[i] = (float)c;
  sin_t[i] = (float)s;
}

// RoPE + QK-norm on one head vector per warp (D = 128): lane l owns the pairs
// (2l, 2l + 64) and (2l + 1, 2l + 65).
template <typename T>
__device__ __forceinline__ void rope_norm_head(const T* src, T* dst, const float* cs, const float* sn,
                                               float alpha, float eps, int lane) {
  const int j = 2 * lane;
  const float a0 = ldf(src + j), a1 = ldf(src + j + 1);
  const float b0 = ldf(src + j + 64), b1 = ldf(src + j + 65);
  const float c0 = cs[j], c1 = cs[j + 1], s0 = sn[j], s1 = sn[j + 1];
  const float y10 = a0 * c0 + b0 * s0, y11 = a1 * c1 + b1 * s1;
  const float y20 = -a0 * s0 + b0 * c0, y21 = -a1 * s1 + b1 * c1;
  float ss = y10 * y10 + y11 * y11 + y20 * y20 + y21 * y21;
  ss = warp_sum(ss);
  const float r = alpha / sqrtf(ss / 128.0f + eps);
  Act<T>::st(dst + j, y10 * r);
  Act<T>::st(dst + j + 1, y11 * r);
  Act<T>::st(dst + j + 64, y20 * r);
  Act<T>::st(dst + j + 65, y21 * r);
}

// In place on the fused qkv buffer [M, ld] = (q heads | k heads | v heads):
// q, k <- alpha RMSNorm(RoPE(.)); v += g * VE[tok] when a table is given.
// One warp per (token, head slot).
template <typename T>
__global__ void k_rope_qknorm_ve(T* qkv, int ld, int T_, int H, int Hkv, int D, const float* cos_t,
                                 const float* sin_t, float alpha, float eps, const int32_t* tokens,
                                 const T* ve, const float* gate, int V, int M) {
  const int lane = threadIdx.x & 31;
  const int slots = H + Hkv + (ve != nullptr ? Hkv : 0);
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= (long long)M * slots) return;
  const int m = (int)(wid / slots);
  const int s = (int)(wid % slots);
  const int t = m % T_;
  T* row = qkv + (size_t)m * ld;
  if (s < H + Hkv) {
    T* u = row + s * D;
    rope_norm_head<T>(u, u, cos_t + (size_t)t * (D / 2), sin_t + (size_t)t * (D / 2), alpha, eps, lane);
  } else {
    const int h = s - H - Hkv;
    T* u = row + (H + Hkv + h) * D;
    int tok = tokens[m];
    tok = min(max(tok, 0), V - 1);
    const T* e = ve + (size_t)tok * Hkv * D + h * D;
    const float g = gate[(size_t)m * Hkv + h];
    for (int j = lane; j < D; j += 32) Act<T>::st(u + j, ldf(u + j) + g * ldf(e + j));
  }
}

// RoPE + QK-norm from separate q/k inputs ([B, T, H, D] contiguous) into qo/ko.
template <typename T>
__global__ void k_rope_qknorm_copy(const T* q, const T* k, T* qo, T* ko, int T_, int H, int Hkv,
                                   int D, const float* cos_t, const float* sin_t, float alpha,
                                   float eps, int M) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int slots = H + Hkv;
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= (long long)M * slots) return;
  const int m = (int)(wid / slots);
  const int s = (int)(wid % slots);
  const int t = m % T_;
  const T* src = s < H ? q + ((size_t)m * H + s) * D : k + ((size_t)m * Hkv + (s - H)) * D;
  T* dst = s < H ? qo + ((size_t)m * H + s) * D : ko + ((size_t)m * Hkv + (s - H)) * D;
  rope_norm_head<T>(src, dst, cos_t + (size_t)t * (D / 2), sin_t + (size_t)t * (D / 2), alpha, eps, lane);
}

// Per-token CE from materialised softcapped logits (fp32 path): one CTA per row.
__global__ void k_ce_rows(const float* logits, int ldl, const int32_t* targets, int V, float* loss,
                          int* status) {
  __shared__ float red[32];
  const int m = blockIdx.x;
  const float* z = logits + (size_t)m * ldl;
  float mx = -INFINITY;
  for (int c = threadIdx.x; c < V; c += blockDim.x) mx = fmaxf(mx, z[c]);
  mx = warp_max(mx);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = -INFINITY;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) mx = fmaxf(mx, red[i]);
  float s = 0.f;
  for (int c = threadIdx.x; c < V; c += blockDim.x) s += expf(z[c] - mx);
  s = block_sum(s, red);
  if (threadIdx.x == 0) {
    int y = targets[m];
    float l = 0.f;
    if (y != -1) {
      if (y < 0 || y >= V) {
        atomicOr(status, kStatusData);
        y = min(max(y, 0), V - 1);
      }
      l = (mx + logf(s)) - z[y];
    }
    loss[m] = l;
  }
}

// Merge per-(row, tile) partial sums sum_n exp(zhat_n - offset) into the
// row's log-sum-exp and subtract the target's zhat.  One warp per row.
__global__ void k_ce_combine(const float* ce_sum, const float* ce_tgt, int n_tiles, float offset,
                             const int32_t* targets, int M, int V, float* loss, int* status) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  const float* ps = ce_sum + (size_t)m * n_tiles;
  float s = 0.f;
  for (int i = lane; i < n_tiles; i += 32) s += ps[i];
  s = warp_sum(s);
  if (lane == 0) {
    const int y = targets[m];
    float l = 0.f;
    if (y != -1) {
      if (y < 0 || y >= V) atomicOr(status, kStatusData);
      l = (offset + logf(s)) - ce_tgt[m];
    }
    loss[m] = l;
  }
}

// Mean of loss over valid targets, fixed reduction order (deterministic).
__global__ void k_loss_mean(const float* loss, const int32_t* targets, int n, float* out) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float rs[32];
  __shared__ float rc[32];
  float s = 0.f, c = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    if (targets[i] != -1) {
      s += loss[i];
      c += 1.f;
    }
  s = warp_sum(s);
  c = warp_sum(c);
  if ((threadIdx.x & 31) == 0) {
    rs[threadIdx.x >> 5] = s;
    rc[threadIdx.x >> 5] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float S = 0.f, Cn = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      S += rs[i];
      Cn += rc[i];
    }
    *out = Cn > 0.f ? S / Cn : __int_as_float(0x7fc00000);
  }
}

}  // namespace

void launch_embed(const void* wte, const int32_t* tokens, const float* smear_gate, int smear,
                  int gate_channels, const float* lam0, const float* mu0, float eps, int B, int T, int C, int V,
                  int act_bf16, float* x, float* x0, bf16* xb, float* ss, int ss_parts, int* status,
                  cudaStream_t st) {
  LaunchScope scope_(KK_EMBED, st);
  const int M = B * T;
  const size_t sh = (size_t)(2 * C + 32) * sizeof(float);
  if (act_bf16)
    launch_pdl(k_embed<bf16>, dim3(M), dim3(256), sh, st, 1, (const bf16*)wte, tokens, smear_gate, smear,
               gate_channels, lam0, mu0, eps, T, C, V, x, x0, xb, ss, ss_parts, status);
  else
    launch_pdl(k_embed<float>, dim3(M), dim3(256), sh, st, 1, (const float*)wte, tokens, smear_gate, smear,
               gate_channels, lam0, mu0, eps, T, C, V, x, x0, xb, ss, ss_parts, status);
}

void launch_rmsnorm(const float* x, void* xn, int M, int C, float eps, int act_bf16,
                    const float* ve_gate, int Hkv, int gate_channels, float gate_scale, float* gate_out,
                    cudaStream_t st) {
  LaunchScope scope_(KK_RMSNORM, st);
  const int warps = 8;
  const int grid = (M + warps - 1) / warps;
  if (act_bf16)
    k_rmsnorm<bf16><<<grid, warps * 32, 0, st>>>(x, (bf16*)xn, M, C, eps, ve_gate, Hkv, gate_channels,
                                                 gate_scale, gate_out);
  else
    k_rmsnorm<float><<<grid, warps * 32, 0, st>>>(x, (float*)xn, M, C, eps, ve_gate, Hkv,
                                                  gate_channels, gate_scale, gate_out);
}

void launch_rope_table(float* cos_t, float* sin_t, int T, int D, float base, cudaStream_t st, float* fsplit,
                       int tbits) {
  LaunchScope scope_(KK_ROPE_TABLE, st);
  const int n = T * (D / 2);
  launch_pdl(k_rope_table, dim3((n + 255) / 256), dim3(256), 0, st, 1, cos_t, sin_t, T, D, (double)base, fsplit,
             tbits);
}

void launch_rope_qknorm_ve(void* qkv, int ld, int B, int T, int H, int Hkv, int D,
                           const float* cos_t, const float* sin_t, float alpha, float eps,
                           const int32_t* tokens, const void* ve, const float* gate, int V,
                           int act_bf16, int* status, cudaStream_t st) {
  LaunchScope scope_(KK_ROPE_QKNORM, st);
  (void)status;
  const int M = B * T;
  const int slots = H + Hkv + (ve != nullptr ? Hkv : 0);
  const long long warps = (long long)M * slots;
  const int wpb = 8;
  const unsigned grid = (unsigned)((warps + wpb - 1) / wpb);
  if (act_bf16)
    k_rope_qknorm_ve<bf16><<<grid, wpb * 32, 0, st>>>((bf16*)qkv, ld, T, H, Hkv, D, cos_t, sin_t, alpha,
                                                      eps, tokens, (const bf16*)ve, gate, V, M);
  else
    k_rope_qknorm_ve<float><<<grid, wpb * 32, 0, st>>>((float*)qkv, ld, T, H, Hkv, D, cos_t, sin_t,
                                                       alpha, eps, tokens, (const float*)ve, gate, V, M);
}

void launch_rope_qknorm_copy(const void* q, const void* k, void* qo, void* ko, int B, int T, int H,
                             int Hkv, int D, const float* cos_t, const float* sin_t, float alpha,
                             float eps, int act_bf16, cudaStream_t st) {
  LaunchScope scope_(KK_ROPE_QKNORM, st);
  const int M = B * T;
  const long long warps = (long long)M * (H + Hkv);
  const int wpb = 8;
  const unsigned grid = (unsigned)((warps + wpb - 1) / wpb);
  if (act_bf16)
    launch_pdl(k_rope_qknorm_copy<bf16>, dim3(grid), dim3(wpb * 32), 0, st, 1, (const bf16*)q, (const bf16*)k,
               (bf16*)qo, (bf16*)ko, T, H, Hkv, D, cos_t, sin_t, alpha, eps, M);
  else
    launch_pdl(k_rope_qknorm_copy<float>, dim3(grid), dim3(wpb * 32), 0, st, 1, (const float*)q,
               (const float*)k, (float*)qo, (float*)ko, T, H, Hkv, D, cos_t, sin_t, alpha, eps, M);
}

void launch_ce_rows(const float* logits, int ldl, const int32_t* targets, int M, int V, float* loss,
                    int* status, cudaStream_t st) {
  LaunchScope scope_(KK_CE_ROWS, st);
  k_ce_rows<<<M, 256, 0, st>>>(logits, ldl, targets, V, loss, status);
}

void launch_ce_combine(const float* ce_sum, const float* ce_tgt, int n_tiles, float offset,
                       const int32_t* targets, int M, int V, float* loss, int* status, cudaStream_t st) {
  LaunchScope scope_(KK_CE_COMBINE, st);
  const int wpb = 8;
  launch_pdl(k_ce_combine, dim3((M + wpb - 1) / wpb), dim3(wpb * 32), 0, st, 1, ce_sum, ce_tgt, n_tiles, offset,
             targets, M, V, loss, status);
}

void launch_loss_mean(const float* loss, const int32_t* targets, int n, float* out, cudaStream_t st) {
  LaunchScope scope_(KK_LOSS_MEAN, st);
  launch_pdl(k_loss_mean, dim3(1), dim3(1024), 0, st, 1, loss, targets, n, out);
}

}  // namespace nc
