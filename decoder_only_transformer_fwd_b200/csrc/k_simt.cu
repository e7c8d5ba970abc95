// CUDA-core GEMM and attention: the fp32 debug path (exact expf/tanhf, fp32
// FFMA) and a cross-check for the tensor-core path in bf16 mode.
#include "epilogue.cuh"

namespace nc {

namespace {

template <typename T>
__device__ __forceinline__ float ldf(const T* p) { return Act<T>::ld(p); }

// C[M, N] = A[M, K] B[N, K]^T; 64x64 tile, 16-deep k-slices, 4x4 per thread.
template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T* __restrict__ A, int lda,
                                                   const T* __restrict__ Bm, int ldb, int M, int N,
                                                   int K, EpiParams ep) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int lr = tid >> 2, lc = (tid & 3) * 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + lr, n = n0 + lr, k = k0 + lc + i;
      As[lc + i][lr] = (m < M && k < K) ? ldf(A + (size_t)m * lda + k) : 0.f;
      Bs[lc + i][lr] = (n < N && k < K) ? ldf(Bm + (size_t)n * ldb + k) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) epi_apply<T>(ep, m, n, acc[i][j]);
    }
}

// Windowed causal attention, 64 queries x one head per CTA, online softmax
// over 64-key tiles ("The Mathematics of Karpathy's nanochat", §Scaled
// Dot-Product Attention with Sliding Window).  D = 128.
constexpr int kAQ = 64, kAK = 64, kAD = 128;

template <typename T>
__global__ void __launch_bounds__(256) k_attn_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                   const T* __restrict__ v, int ldq, int ldk, int ldv,
                                                   T* __restrict__ o, int ldo, int T_, int H, int Hkv,
                                                   int window, float scale) {
  extern __shared__ float sm[];
  float* Qs = sm;                          // [D][65]   (transposed)
  float* Ks = Qs + kAD * 65;               // [D][65]   (transposed)
  float* Vs = Ks + kAD * 65;               // [64][128]
  float* Ps = Vs + kAK * kAD;              // [64 keys][65] (transposed)
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int q0 = blockIdx.x * kAQ;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (H / Hkv);
  const size_t rowbase = (size_t)b * T_;

  for (int e = tid; e < kAQ * kAD; e += 256) {
    const int i = e / kAD, d = e % kAD;
    const int t = q0 + i;
    Qs[d * 65 + i] = t < T_ ? ldf(q + (rowbase + t) * ldq + h * kAD + d) : 0.f;
  }
  float mrow[4], lrow[4], acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mrow[i] = -INFINITY;
    lrow[i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  }
  const int lo = max(0, q0 - window + 1);
  const int hi = min(q0 + kAQ - 1, T_ - 1);
  for (int kt = lo / kAK; kt <= hi / kAK; ++kt) {
    const int k0 = kt * kAK;
    __syncthreads();
    for (int e = tid; e < kAK * kAD; e += 256) {
      const int j = e / kAD, d = e % kAD;
      const int t = k0 + j;
      const bool ok = t < T_;
      Ks[d * 65 + j] = ok ? ldf(k + (rowbase + t) * ldk + hk * kAD + d) : 0.f;
      Vs[j * kAD + d] = ok ? ldf(v + (rowbase + t) * ldv + hk * kAD + d) : 0.f;
    }
    __syncthreads();
    float s[4][4] = {};
    for (int d = 0; d < kAD; ++d) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = Qs[d * 65 + ty * 4 + i];
        bb[i] = Ks[d * 65 + tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = fmaf(a[i], bb[j], s[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qi = q0 + ty * 4 + i;
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kj = k0 + tx * 4 + j;
        const bool vis = kj <= qi && qi - kj < window && kj < T_;
        s[i][j] = vis ? s[i][j] * scale : -INFINITY;
        tmax = fmaxf(tmax, s[i][j]);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      const float mnew = fmaxf(mrow[i], tmax);
      const float corr = (mnew == -INFINITY) ? 1.f : expf(mrow[i] - mnew);
      float psum = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = (mnew == -INFINITY) ? 0.f : expf(s[i][j] - mnew);
        psum += p;
        Ps[(tx * 4 + j) * 65 + ty * 4 + i] = p;
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      lrow[i] = lrow[i] * corr + psum;
      mrow[i] = mnew;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] *= corr;
    }
    __syncthreads();
    for (int j = 0; j < kAK; ++j) {
      float p[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) p[i] = Ps[j * 65 + ty * 4 + i];
      float vv[8];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        vv[c] = Vs[j * kAD + tx * 4 + c];
        vv[4 + c] = Vs[j * kAD + 64 + tx * 4 + c];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = fmaf(p[i], vv[c], acc[i][c]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qi = q0 + ty * 4 + i;
    if (qi >= T_) continue;
    const float inv = 1.0f / lrow[i];
    T* dst = o + (rowbase + qi) * ldo + h * kAD;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      Act<T>::st(dst + tx * 4 + c, acc[i][c] * inv);
      Act<T>::st(dst + 64 + tx * 4 + c, acc[i][4 + c] * inv);
    }
  }
}

}  // namespace

void launch_gemm_simt(const void* A, int lda, const void* Bm, int ldb, int M, int N, int K,
                      int act_bf16, const EpiParams& ep, cudaStream_t st) {
  LaunchScope scope_(KK_GEMM_SIMT, st);
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  if (act_bf16)
    k_gemm_simt<bf16><<<grid, 256, 0, st>>>((const bf16*)A, lda, (const bf16*)Bm, ldb, M, N, K, ep);
  else
    k_gemm_simt<float><<<grid, 256, 0, st>>>((const float*)A, lda, (const float*)Bm, ldb, M, N, K, ep);
}

void launch_attn_simt(const void* q, const void* k, const void* v, int ldq, int ldk, int ldv,
                      void* o, int ldo, int B, int T, int H, int Hkv, int window, float scale,
                      int act_bf16, cudaStream_t st) {
  LaunchScope scope_(KK_ATTN_SIMT, st);
  const size_t sh = (size_t)(2 * kAD * 65 + kAK * kAD + kAK * 65) * sizeof(float);
  dim3 grid((T + kAQ - 1) / kAQ, H, B);
  if (act_bf16) {
    if (!smem_optin(k_attn_simt<bf16>, (int)sh)) return;
    k_attn_simt<bf16><<<grid, 256, sh, st>>>((const bf16*)q, (const bf16*)k, (const bf16*)v, ldq, ldk,
                                             ldv, (bf16*)o, ldo, T, H, Hkv, window, scale);
  } else {
    if (!smem_optin(k_attn_simt<float>, (int)sh)) return;
    k_attn_simt<float><<<grid, 256, sh, st>>>((const float*)q, (const float*)k, (const float*)v, ldq,
                                              ldk, ldv, (float*)o, ldo, T, H, Hkv, window, scale);
  }
}

}  // namespace nc
