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

// bf16 tables, C = 32 * EPL: one warp walks a run of `run` (<= 32)
// consecutive positions of one row; lane i loads the run's i-th token id up
// front, so no row load waits for its id.  Lane l holds elements [4 (k * 32 + l), + 4) of every
// row for k < EPL / 4, so each warp-wide access is contiguous: 256 bytes of a
// bf16 row, 512 bytes of an fp32 row.  The next position's embedding row is
// requested before the current one is normalised and stored, so a warp keeps
// two rows of loads in flight; the normalised embedding of the previous
// position is carried in registers (it is what smear mixes in).  Same
// outputs as k_embed: x0, x = (lam0 + mu0) x0, bf16(x) and its sum of squares.
template <int EPL>
__global__ void __launch_bounds__(64) k_embed_vec(
    const bf16* __restrict__ wte, const int32_t* __restrict__ tokens, const float* __restrict__ smear_gate,
    int smear, int gc, const float* __restrict__ lam0p, const float* __restrict__ mu0p, float eps, int B, int T_,
    int C, int V, int run, float* __restrict__ x, float* __restrict__ x0, bf16* __restrict__ xb,
    float* __restrict__ ss, int ss_parts, int* status) {
  constexpr int NCH = EPL / 4;
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int runs_per_row = (T_ + run - 1) / run;
  if (wid >= B * runs_per_row) return;
  const int b = wid / runs_per_row;
  const int t0 = (wid % runs_per_row) * run;
  const int t1 = min(T_, t0 + run);
  const float inv_c = 1.0f / (float)C;
  auto load_raw = [&](int tok, uint2 (&u)[NCH]) {
    const uint2* row = reinterpret_cast<const uint2*>(wte + (size_t)tok * C);
#pragma unroll
    for (int k = 0; k < NCH; ++k) u[k] = row[k * 32 + lane];
  };
  // raw row -> normalised fp32 values
  auto normalise = [&](const uint2 (&u)[NCH], float (&v)[EPL]) {
    float sq = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[k].x));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[k].y));
      v[4 * k] = f0.x;
      v[4 * k + 1] = f0.y;
      v[4 * k + 2] = f1.x;
      v[4 * k + 3] = f1.y;
      sq = fmaf(f0.x, f0.x, fmaf(f0.y, f0.y, fmaf(f1.x, f1.x, fmaf(f1.y, f1.y, sq))));
    }
    const float r = 1.0f / sqrtf(warp_sum(sq) * inv_c + eps);
#pragma unroll
    for (int i = 0; i < EPL; ++i) v[i] *= r;
  };
  int my_tok = 0;  // lane i: the id at position t0 + i, clamped
  if (lane < t1 - t0) {
    my_tok = tokens[(size_t)b * T_ + t0 + lane];
    if (my_tok < 0 || my_tok >= V) {
      atomicOr(status, kStatusData);
      my_tok = min(max(my_tok, 0), V - 1);
    }
  }
  auto token = [&](int t) { return __shfl_sync(0xffffffffu, my_tok, t - t0); };
  float prev[EPL];
  uint2 raw[NCH], nxt[NCH];
  if (smear && t0 > 0) {
    // its out-of-range flag is raised by the warp that owns that position
    const int tp = tokens[(size_t)b * T_ + t0 - 1];
    load_raw(min(max(tp, 0), V - 1), raw);
    normalise(raw, prev);
  }
  load_raw(token(t0), raw);
  const float scale = *lam0p + *mu0p;
  for (int t = t0; t < t1; ++t) {
    if (t + 1 < t1) load_raw(token(t + 1), nxt);  // in flight while this position is processed
    float cur[EPL];
    normalise(raw, cur);
    float g = 0.f;
    if (smear && t > 0) {
      float d = 0.f;
#pragma unroll
      for (int k = 0; k < NCH; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = (k * 32 + lane) * 4 + i;
          if (c < gc) d = fmaf(smear_gate[c], cur[4 * k + i], d);
        }
      g = sigmoidf_(warp_sum(d));
    }
    const size_t m = (size_t)b * T_ + t;
    float sq = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int e0 = (k * 32 + lane) * 4;
      float o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[i] = (smear && t > 0) ? fmaf(g, prev[4 * k + i], cur[4 * k + i]) : cur[4 * k + i];
        prev[4 * k + i] = cur[4 * k + i];
      }
      *reinterpret_cast<float4*>(x0 + m * C + e0) = make_float4(o[0], o[1], o[2], o[3]);
      const float4 xv = make_float4(scale * o[0], scale * o[1], scale * o[2], scale * o[3]);
      *reinterpret_cast<float4*>(x + m * C + e0) = xv;
      sq = fmaf(xv.x, xv.x, fmaf(xv.y, xv.y, fmaf(xv.z, xv.z, fmaf(xv.w, xv.w, sq))));
      if (xb != nullptr) {
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(xv.x, xv.y), b1 = __floats2bfloat162_rn(xv.z, xv.w);
        *reinterpret_cast<uint2*>(xb + m * C + e0) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
      }
    }
    if (xb != nullptr) {
      // the first block's norm input: sum of squares in slot 0, other slots 0
      sq = warp_sum(sq);
      for (int j = lane; j < ss_parts; j += 32) ss[m * ss_parts + j] = j == 0 ? sq : 0.f;
    }
#pragma unroll
    for (int k = 0; k < NCH; ++k) raw[k] = nxt[k];
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

// The same for bf16 q/k with 16-byte accesses: eight lanes per head vector,
// lane i holding elements [8 i, 8 i + 8) of each half (so the pairs (j, j + 64)
// it rotates are its own), the sum of squares reduced over the eight lanes.
// A warp covers four head vectors.
__global__ void __launch_bounds__(256) k_rope_qknorm_copy_bf16(
    const bf16* __restrict__ q, const bf16* __restrict__ k, bf16* __restrict__ qo, bf16* __restrict__ ko, int T_,
    int H, int Hkv, const float* __restrict__ cos_t, const float* __restrict__ sin_t, float alpha, float eps,
    int M) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int slots = H + Hkv;
  const long long hv = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4 + (lane >> 3);
  const bool valid = hv < (long long)M * slots;
  const int m = valid ? (int)(hv / slots) : 0;
  const int s = valid ? (int)(hv % slots) : 0;
  const int t = m % T_;
  const int i8 = (lane & 7) * 8;
  const bf16* src = s < H ? q + ((size_t)m * H + s) * 128 : k + ((size_t)m * Hkv + (s - H)) * 128;
  bf16* dst = s < H ? qo + ((size_t)m * H + s) * 128 : ko + ((size_t)m * Hkv + (s - H)) * 128;
  float a[8], bb[8], cs[8], sn[8];
  if (valid) {
    const uint4 ua = *reinterpret_cast<const uint4*>(src + i8);
    const uint4 ub = *reinterpret_cast<const uint4*>(src + 64 + i8);
    const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[i]));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[i]));
      a[2 * i] = fa.x;
      a[2 * i + 1] = fa.y;
      bb[2 * i] = fb.x;
      bb[2 * i + 1] = fb.y;
    }
    const float4* c4 = reinterpret_cast<const float4*>(cos_t + (size_t)t * 64 + i8);
    const float4* s4 = reinterpret_cast<const float4*>(sin_t + (size_t)t * 64 + i8);
    const float4 c0 = c4[0], c1 = c4[1], s0 = s4[0], s1 = s4[1];
    const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cs[i] = cv[i];
      sn[i] = sv[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = bb[i] = cs[i] = sn[i] = 0.f;
  }
  float y1[8], y2[8], ssq = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    y1[i] = a[i] * cs[i] + bb[i] * sn[i];
    y2[i] = -a[i] * sn[i] + bb[i] * cs[i];
    ssq = fmaf(y1[i], y1[i], fmaf(y2[i], y2[i], ssq));
  }
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 1);
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 2);
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 4);
  const float r = alpha / sqrtf(ssq / 128.0f + eps);
  if (valid) {
    uint32_t w1[4], w2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 p1 = __floats2bfloat162_rn(y1[2 * i] * r, y1[2 * i + 1] * r);
      const __nv_bfloat162 p2 = __floats2bfloat162_rn(y2[2 * i] * r, y2[2 * i + 1] * r);
      w1[i] = *reinterpret_cast<const uint32_t*>(&p1);
      w2[i] = *reinterpret_cast<const uint32_t*>(&p2);
    }
    *reinterpret_cast<uint4*>(dst + i8) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
    *reinterpret_cast<uint4*>(dst + 64 + i8) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
  }
}

// out = bf16(g * in) over n elements (n % 8 == 0), 16-byte accesses.
__global__ void k_scale_bf16(const bf16* __restrict__ in, bf16* __restrict__ out, long long n8, float g) {
  pdl_launch_dependents();
  pdl_wait();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(in)[i];
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      const __nv_bfloat162 b = __floats2bfloat162_rn(g * f.x, g * f.y);
      w[j] = *reinterpret_cast<const uint32_t*>(&b);
    }
    reinterpret_cast<uint4*>(out)[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
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
                             const int32_t* targets, int M, int V, float* loss, float* lse, int* status) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  const float* ps = ce_sum + (size_t)m * n_tiles;
  float s = 0.f;
  if ((n_tiles & 3) == 0) {
    // 16-byte loads: a row of 2 V_pad / 128 partial sums is 2 KB at V = 32768
    const float4* p4 = reinterpret_cast<const float4*>(ps);
#pragma unroll 4
    for (int i = lane; i < n_tiles / 4; i += 32) {
      const float4 v = p4[i];
      s += (v.x + v.y) + (v.z + v.w);
    }
  } else {
    for (int i = lane; i < n_tiles; i += 32) s += ps[i];
  }
  s = warp_sum(s);
  if (lane == 0) {
    const int y = targets[m];
    const float row_lse = offset + logf(s);
    float l = 0.f;
    if (y != -1) {
      if (y < 0 || y >= V) atomicOr(status, kStatusData);
      l = row_lse - ce_tgt[m];
    }
    loss[m] = l;
    if (lse != nullptr) lse[m] = row_lse;
  }
}

// 1 / (number of targets != -1), 0 when there is none.  One CTA.
__global__ void k_inv_count(const int32_t* targets, int n, float* inv_count) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int part[32];
  int c = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) c += targets[i] != -1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int total = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) total += part[i];
    *inv_count = total > 0 ? 1.0f / (float)total : 0.f;
  }
}

// RMSNorm backward ("The Mathematics of Karpathy's nanochat", §RMS
// Normalization: xn = x r, r = (mean(x^2) + eps)^(-1/2)): with g = r dL/dxn,
// dL/dx = r dL/dxn - x r^3 (x . dL/dxn) / C = g - x r^2 (x . g) / C.  One warp
// per row, 16-byte accesses (C % 4 == 0).
__global__ void k_rmsnorm_bwd(const float* __restrict__ x, const float* __restrict__ g, float* __restrict__ dx,
                              int M, int C, float eps) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)m * C);
  const float4* gr = reinterpret_cast<const float4*>(g + (size_t)m * C);
  float ss = 0.f, xg = 0.f;
  for (int i = lane; i < C / 4; i += 32) {
    const float4 a = xr[i], b = gr[i];
    ss = fmaf(a.x, a.x, fmaf(a.y, a.y, fmaf(a.z, a.z, fmaf(a.w, a.w, ss))));
    xg = fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, xg))));
  }
  ss = warp_sum(ss);
  xg = warp_sum(xg);
  const float k = xg / (ss + eps * (float)C);  // r^2 (x . g) / C
  float4* dr = reinterpret_cast<float4*>(dx + (size_t)m * C);
  for (int i = lane; i < C / 4; i += 32) {
    const float4 a = xr[i], b = gr[i];
    dr[i] = make_float4(b.x - k * a.x, b.y - k * a.y, b.z - k * a.z, b.w - k * a.w);
  }
}

// PrefixRMSNorm ("Fully Nested Transformers" README: normalisation that does
// not leak information backward down the hierarchy): block a of row m, the
// columns [end[a-1], end[a]), is divided by the RMS of the row's prefix
// [0, end[a]).  One warp per row: the prefix sums of squares first (16-byte
// loads, one warp reduction per block), then every block scaled and stored.
template <typename TO>
__global__ void k_prefix_rmsnorm(const float* __restrict__ x, int M, int C, PrefixBlocks pb, float eps,
                                 TO* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)m * C);
  float inv[kMaxPrefixBlocks];
  float cum = 0.f;
  int c0 = 0;
#pragma unroll
  for (int a = 0; a < kMaxPrefixBlocks; ++a) {
    if (a < pb.k) {
      float ss = 0.f;
      for (int i = c0 / 4 + lane; i < pb.end[a] / 4; i += 32) {
        const float4 v = xr[i];
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
      }
      cum += warp_sum(ss);
      inv[a] = rsqrtf(cum / (float)pb.end[a] + eps);
      c0 = pb.end[a];
    }
  }
  c0 = 0;
#pragma unroll
  for (int a = 0; a < kMaxPrefixBlocks; ++a) {
    if (a < pb.k) {
      const float r = inv[a];
      for (int i = c0 / 4 + lane; i < pb.end[a] / 4; i += 32) {
        const float4 v = xr[i];
        const float4 y = make_float4(v.x * r, v.y * r, v.z * r, v.w * r);
        if constexpr (sizeof(TO) == 2) {
          const __nv_bfloat162 b0 = __floats2bfloat162_rn(y.x, y.y), b1 = __floats2bfloat162_rn(y.z, y.w);
          reinterpret_cast<uint2*>(out + (size_t)m * C)[i] =
              make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
        } else {
          reinterpret_cast<float4*>(out + (size_t)m * C)[i] = y;
        }
      }
      c0 = pb.end[a];
    }
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
  if (act_bf16 && C % 128 == 0 && C <= 2048) {
    constexpr int kRun = 8;
    const int warps = B * ((T + kRun - 1) / kRun);
    const dim3 grid((warps + 1) / 2), block(64);
    const bf16* w = (const bf16*)wte;
    switch (C / 32) {
#define NC_EMBED_CASE(E)                                                                                      \
  case E:                                                                                                     \
    launch_pdl(k_embed_vec<E>, grid, block, 0, st, 1, w, tokens, smear_gate, smear, gate_channels, lam0, mu0, \
               eps, B, T, C, V, kRun, x, x0, xb, ss, ss_parts, status);                                       \
    return;
      NC_EMBED_CASE(4) NC_EMBED_CASE(8) NC_EMBED_CASE(12) NC_EMBED_CASE(16) NC_EMBED_CASE(20) NC_EMBED_CASE(24)
      NC_EMBED_CASE(28) NC_EMBED_CASE(32) NC_EMBED_CASE(36) NC_EMBED_CASE(40) NC_EMBED_CASE(44) NC_EMBED_CASE(48)
      NC_EMBED_CASE(52) NC_EMBED_CASE(56) NC_EMBED_CASE(60) NC_EMBED_CASE(64)
#undef NC_EMBED_CASE
      default: break;
    }
  }
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
  const int n = T * (D / 2);  // T = 0: the split frequencies only
  launch_pdl(k_rope_table, dim3(n > 0 ? (n + 255) / 256 : 1), dim3(256), 0, st, 1, cos_t, sin_t, T, D, (double)base,
             fsplit, tbits);
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
  if (act_bf16 && D == 128) {
    const long long vwarps = (warps + 3) / 4;  // four head vectors per warp
    launch_pdl(k_rope_qknorm_copy_bf16, dim3((unsigned)((vwarps + wpb - 1) / wpb)), dim3(wpb * 32), 0, st, 1,
               (const bf16*)q, (const bf16*)k, (bf16*)qo, (bf16*)ko, T, H, Hkv, cos_t, sin_t, alpha, eps, M);
    return;
  }
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
                       const int32_t* targets, int M, int V, float* loss, float* lse, int* status, cudaStream_t st) {
  LaunchScope scope_(KK_CE_COMBINE, st);
  const int wpb = 8;
  launch_pdl(k_ce_combine, dim3((M + wpb - 1) / wpb), dim3(wpb * 32), 0, st, 1, ce_sum, ce_tgt, n_tiles, offset,
             targets, M, V, loss, lse, status);
}

void launch_scale_bf16(const bf16* in, bf16* out, long long n, float g, int num_sms, cudaStream_t st) {
  LaunchScope scope_(KK_ROPE_QKNORM, st);
  const long long n8 = n / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks > 8LL * num_sms) blocks = 8LL * num_sms;
  if (blocks < 1) blocks = 1;
  launch_pdl(k_scale_bf16, dim3((unsigned)blocks), dim3(256), 0, st, 1, in, out, n8, g);
}

void launch_inv_count(const int32_t* targets, int n, float* inv_count, cudaStream_t st) {
  LaunchScope scope_(KK_HEAD_BWD_ROWS, st);
  launch_pdl(k_inv_count, dim3(1), dim3(1024), 0, st, 1, targets, n, inv_count);
}

void launch_rmsnorm_bwd(const float* x, const float* g, float* dx, int M, int C, float eps, cudaStream_t st) {
  LaunchScope scope_(KK_HEAD_BWD_ROWS, st);
  const int wpb = 8;
  launch_pdl(k_rmsnorm_bwd, dim3((M + wpb - 1) / wpb), dim3(wpb * 32), 0, st, 1, x, g, dx, M, C, eps);
}

void launch_prefix_rmsnorm(const float* x, int M, int C, const PrefixBlocks& pb, float eps, void* out, int out_bf16,
                           cudaStream_t st) {
  LaunchScope scope_(KK_PREFIX_NORM, st);
  constexpr int wpb = 8;
  const dim3 grid((M + wpb - 1) / wpb), block(wpb * 32);
  if (out_bf16)
    launch_pdl(k_prefix_rmsnorm<bf16>, grid, block, 0, st, 1, x, M, C, pb, eps, static_cast<bf16*>(out));
  else
    launch_pdl(k_prefix_rmsnorm<float>, grid, block, 0, st, 1, x, M, C, pb, eps, static_cast<float*>(out));
}

void launch_loss_mean(const float* loss, const int32_t* targets, int n, float* out, cudaStream_t st) {
  LaunchScope scope_(KK_LOSS_MEAN, st);
  launch_pdl(k_loss_mean, dim3(1), dim3(1024), 0, st, 1, loss, targets, n, out);
}

}  // namespace nc
