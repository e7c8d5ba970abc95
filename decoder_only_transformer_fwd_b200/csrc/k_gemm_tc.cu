// tcgen05 GEMM for sm_100a: C[M, N] = A[M, K] B[N, K]^T with bf16 operands
// and fp32 accumulation in tensor memory, followed by a fused epilogue.
//
// Structure (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: A and B k-slices (64 wide, 128-byte swizzle)
//               into a STAGES-deep shared-memory ring;
//   warp 1      allocates 2*BN TMEM columns; one thread issues tcgen05.mma
//               (M = 128, N = BN, K = 16) into one of two accumulators;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one TMEM lane per
//               output row), the fused element-wise op, global stores.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i + 1.  Every wait is bounded (see ptx::mbar_wait); on a timeout the CTA
// records NC_ERR_TIMEOUT, stops issuing work, waits for its own copies and
// MMAs, frees its TMEM and returns.
//
// Fused epilogues ("The Mathematics of Karpathy's nanochat"): ReLU^2
// (§Feed-Forward Network), residual updates with x0 re-injection and backout
// (§Residual Stream with Learnable Scalars; backout per the "nanochat depth
// sweep" card), and for the head the softcap 15 tanh(z/15) (§Logit Softcap)
// with a streaming log-sum-exp for the cross-entropy (§Cross-Entropy Loss):
// per (row, tile) it stores sum_n exp(zhat_n - cap) (zhat <= cap, so the sum
// is bounded without a running max) and the target's zhat, never the logits
// unless asked.
#include <cudaTypedefs.h>

#include <mutex>

#include "epilogue.cuh"
#include "ptx.cuh"

namespace nc {

namespace {

constexpr int kBM = 128, kBK = 64, kUK = 16;

template <int BN>
struct TcCfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int NBARS = 2 * STAGES + 5;
  // per epilogue warp: a 32 x 32 fp32 transpose buffer (row pitch 33)
  static constexpr int STAGE_FLOATS = 32 * 33;
  static constexpr int EPI_BYTES = 4 * STAGE_FLOATS * 4;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256 + EPI_BYTES;
};

struct TcArgs {
  int M, N, K;
  int tiles_m, tiles_n, num_tiles;
  int* status;
};

__device__ __forceinline__ float bits2f(uint32_t u) { return __uint_as_float(u); }

// Softcap via tanh(u) = 1 - 2 / (exp(2u) + 1).
__device__ __forceinline__ float softcap_fast(float z, float cap) {
  const float t = __expf(2.0f * z / cap);
  return cap * (1.0f - 2.0f / (t + 1.0f));
}

// Epilogue for 32 consecutive columns [n, n + 32) of row m held in r[].
__device__ __forceinline__ void epi_chunk(const EpiParams& ep, const TcArgs& a, int m, int n,
                                          const uint32_t (&r)[32], float& ce_sum, float& ce_tgt,
                                          int y) {
  const bool row_ok = m < a.M;
  switch (ep.mode) {
    case EPI_STORE:
    case EPI_RELU2: {
      if (!row_ok) return;
      bf16* dst = reinterpret_cast<bf16*>(ep.out) + (size_t)m * ep.ldo + n;
      if (n + 32 <= a.N) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v0 = bits2f(r[q * 8 + 2 * e]), v1 = bits2f(r[q * 8 + 2 * e + 1]);
            if (ep.mode == EPI_RELU2) {
              v0 = fmaxf(v0, 0.f); v0 *= v0;
              v1 = fmaxf(v1, 0.f); v1 *= v1;
            }
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
            w[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          d4[q] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (n + i < a.N) epi_apply<bf16>(ep, m, n + i, bits2f(r[i]));
      }
    } break;
    case EPI_RESID:
    case EPI_BLOCK_END: {
      if (!row_ok) return;
      if (n + 32 <= a.N) {
        float4* x4 = reinterpret_cast<float4*>(ep.x + (size_t)m * ep.ldx + n);
        const float4* x04 = reinterpret_cast<const float4*>(ep.x0 + (size_t)m * ep.ldx + n);
        float4* b4 = reinterpret_cast<float4*>(ep.xbo + (size_t)m * ep.ldx + n);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 v = x4[q];
          v.x += bits2f(r[4 * q + 0]);
          v.y += bits2f(r[4 * q + 1]);
          v.z += bits2f(r[4 * q + 2]);
          v.w += bits2f(r[4 * q + 3]);
          if (ep.mode == EPI_BLOCK_END) {
            if (ep.capture_bo) b4[q] = v;
            if (ep.end_kind == 1) {
              const float4 z = x04[q];
              const float lam = *ep.lam, mu = *ep.mu;
              v.x = lam * v.x + mu * z.x;
              v.y = lam * v.y + mu * z.y;
              v.z = lam * v.z + mu * z.z;
              v.w = lam * v.w + mu * z.w;
            } else if (ep.end_kind == 2) {
              const float4 z = b4[q];
              v.x -= ep.beta * z.x;
              v.y -= ep.beta * z.y;
              v.z -= ep.beta * z.z;
              v.w -= ep.beta * z.w;
            }
          }
          x4[q] = v;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (n + i < a.N) epi_apply<float>(ep, m, n + i, bits2f(r[i]));
      }
    } break;
    case EPI_CE: {
      float zh[32];
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        zh[i] = softcap_fast(bits2f(r[i]), ep.cap);
        const bool ok = (n + i) < ep.vocab;
        s += ok ? __expf(zh[i] - ep.cap) : 0.f;
        if (n + i == y) ce_tgt = zh[i];
      }
      ce_sum += s;
      if (row_ok && ep.logits != nullptr) {
        float* dst = ep.logits + (size_t)m * ep.ldl + n;
        if (n + 32 <= ep.vocab) {
          float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
          for (int q = 0; q < 8; ++q) d4[q] = make_float4(zh[4 * q], zh[4 * q + 1], zh[4 * q + 2], zh[4 * q + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (n + i < ep.vocab) dst[i] = zh[i];
        }
      }
    } break;
    default:
      break;
  }
}

// Residual epilogues (EPI_RESID, EPI_BLOCK_END) for a 32-row x 32-column
// chunk: the warp's rows arrive one per lane (TMEM lane = row); they are
// transposed through shared memory so that for each row the warp reads and
// writes one contiguous 128-byte segment of x (and x0 / x_bo), with all the
// chunk's loads issued before its stores.
__device__ __forceinline__ void epi_resid_chunk(const EpiParams& ep, const TcArgs& a, float* stage,
                                                int row0, int n, const uint32_t (&r)[32], int lane) {
#pragma unroll
  for (int i = 0; i < 32; ++i) stage[lane * 33 + i] = __uint_as_float(r[i]);
  __syncwarp();
  const int col = n + lane;
  const bool col_ok = col < a.N;
  float acc[32], xv[32], zv[32];
#pragma unroll
  for (int rr = 0; rr < 32; ++rr) acc[rr] = stage[rr * 33 + lane];
  __syncwarp();
  const bool bend = ep.mode == EPI_BLOCK_END;
  const bool need_x0 = bend && ep.end_kind == 1;
  const bool need_bo = bend && ep.end_kind == 2 && !ep.capture_bo;
#pragma unroll
  for (int rr = 0; rr < 32; ++rr) {
    const int m = row0 + rr;
    const size_t i = (size_t)m * ep.ldx + col;
    const bool ok = col_ok && m < a.M;
    xv[rr] = ok ? ep.x[i] : 0.f;
    zv[rr] = (ok && need_x0) ? ep.x0[i] : ((ok && need_bo) ? ep.xbo[i] : 0.f);
  }
  float lam = 1.f, mu = 0.f;
  if (need_x0) {
    lam = *ep.lam;
    mu = *ep.mu;
  }
#pragma unroll
  for (int rr = 0; rr < 32; ++rr) {
    const int m = row0 + rr;
    if (!col_ok || m >= a.M) continue;
    const size_t i = (size_t)m * ep.ldx + col;
    float v = xv[rr] + acc[rr];
    if (bend) {
      if (ep.capture_bo) ep.xbo[i] = v;
      if (ep.end_kind == 1)
        v = lam * v + mu * zv[rr];
      else if (ep.end_kind == 2)
        v = v - ep.beta * (ep.capture_bo ? v : zv[rr]);
    }
    ep.x[i] = v;
  }
}

// Fused QKV epilogue for the 128 columns of one head held in TMEM at taddr:
// q and k heads get RoPE (position m % T) and alpha * RMSNorm over the head;
// v heads get gate * VE[tok] added; one bf16 rounding at the store.
// ("The Mathematics of Karpathy's nanochat", §Rotary Position Embeddings,
// §QK-Norm with Sharpening, §Value Embeddings.)
__device__ __forceinline__ void epi_qkv_head(const EpiParams& ep, const TcArgs& a, uint32_t taddr, int m,
                                             int col0) {
  float x[128];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t u[32];
    ptx::tmem_ld32(taddr + (uint32_t)(c * 32), u);
    ptx::tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(u[i]);
  }
  const bool row_ok = m < a.M;
  if (col0 < ep.qk_cols) {
    const int t = m % ep.T;
    const float4* cs = reinterpret_cast<const float4*>(ep.rope_cos + (size_t)t * 64);
    const float4* sn = reinterpret_cast<const float4*>(ep.rope_sin + (size_t)t * 64);
    float ss = 0.f;
#pragma unroll
    for (int j4 = 0; j4 < 16; ++j4) {
      const float4 c4 = cs[j4], s4 = sn[j4];
      const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * j4 + e;
        const float u1 = x[j], u2 = x[j + 64];
        const float y1 = u1 * cc[e] + u2 * sv[e];
        const float y2 = -u1 * sv[e] + u2 * cc[e];
        x[j] = y1;
        x[j + 64] = y2;
        ss += y1 * y1 + y2 * y2;
      }
    }
    const float r = ep.qk_alpha / sqrtf(ss * (1.0f / 128.0f) + ep.eps);
#pragma unroll
    for (int i = 0; i < 128; ++i) x[i] *= r;
  } else if (ep.ve != nullptr) {
    const int hv = (col0 - ep.qk_cols) >> 7;
    int tok = row_ok ? ep.tokens[m] : 0;
    tok = min(max(tok, 0), ep.vocab - 1);
    const float g = row_ok ? ep.gate[(size_t)m * ep.n_kv_head + hv] : 0.f;
    const uint4* e4 = reinterpret_cast<const uint4*>(reinterpret_cast<const bf16*>(ep.ve) +
                                                     ((size_t)tok * ep.n_kv_head + hv) * 128);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const uint4 w = e4[q];
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ww[e]));
        x[8 * q + 2 * e] += g * f.x;
        x[8 * q + 2 * e + 1] += g * f.y;
      }
    }
  }
  if (!row_ok) return;
  uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(ep.out) + (size_t)m * ep.ldo + col0);
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(x[8 * q + 2 * e], x[8 * q + 2 * e + 1]);
      w[e] = *reinterpret_cast<uint32_t*>(&b2);
    }
    d4[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const TcArgs a, const EpiParams ep) {
  using Cf = TcCfg<BN>;
  constexpr int S = Cf::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cf::STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cf::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_stage = reinterpret_cast<float*>(smem + S * Cf::STAGE_BYTES + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  auto tfull = [&](int i) { return bar0 + 8u * (2 * S + i); };
  auto tempty = [&](int i) { return bar0 + 8u * (2 * S + 2 + i); };
  const uint32_t mma_done = bar0 + 8u * (2 * S + 4);
  auto sA = [&](int s) { return ptx::smem_u32(smem + s * Cf::STAGE_BYTES); };
  auto sB = [&](int s) { return ptx::smem_u32(smem + s * Cf::STAGE_BYTES + Cf::A_BYTES); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(tfull(i), 1);
      ptx::mbar_init(tempty(i), 4);
    }
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), Cf::TMEM_COLS);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nk = a.K / kBK;

  if (warp == 0) {
    if (ptx::elect_one()) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t ph = 0, issued = 0, par = 0;
      for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
        const int mb = tile % a.tiles_m, nb = tile / a.tiles_m;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (*abort_flag || !ptx::mbar_wait(empty(stage), ph ^ 1, a.status)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(full(stage), Cf::STAGE_BYTES);
          ptx::tma_load_2d(sA(stage), &tmA, full(stage), kb * kBK, mb * kBM);
          ptx::tma_load_2d(sB(stage), &tmB, full(stage), kb * kBK, nb * BN);
          issued |= 1u << stage;
          par = (par & ~(1u << stage)) | (ph << stage);
          if (++stage == S) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
      // the copies this thread issued have landed before the CTA may exit
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) ptx::mbar_wait(full(s), (par >> s) & 1, a.status);
    }
  } else if (warp == 1) {
    if (ptx::elect_one()) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = ptx::idesc_bf16(kBM, BN);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
        if (*abort_flag || !ptx::mbar_wait(tempty(acc), aph ^ 1, a.status)) {
          *abort_flag = 1;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (*abort_flag || !ptx::mbar_wait(full(stage), ph, a.status)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t da = ptx::desc_kmajor_sw128(sA(stage));
          const uint64_t db = ptx::desc_kmajor_sw128(sB(stage));
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k)
            ptx::mma_bf16_ss(d, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          ptx::mma_commit(empty(stage));
          if (++stage == S) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        ptx::mma_commit(tfull(acc));
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      // all MMAs of this thread have completed before TMEM is released
      ptx::mma_commit(mma_done);
      ptx::mbar_wait(mma_done, 0, a.status);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int g = warp & 3;  // the TMEM lane quarter this warp may access
    const int row = g * 32 + lane;
    int acc = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      const int mb = tile % a.tiles_m, nb = tile / a.tiles_m;
      if (*abort_flag || !ptx::mbar_wait(tfull(acc), aph, a.status)) {
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const int m = mb * kBM + row;
      const int n0 = nb * BN;
      int y = -1;
      if (ep.mode == EPI_CE && m < a.M) {
        y = ep.targets[m];
        if (y != -1) y = min(max(y, 0), ep.vocab - 1);  // out-of-range ids are flagged by the combine
      }
      float ce_sum = 0.f, ce_tgt = 0.f;
      const uint32_t taddr = tmem + ((uint32_t)(g * 32) << 16) + (uint32_t)(acc * BN);
      if (ep.mode == EPI_QKV) {
#pragma unroll 1
        for (int hh = 0; hh < BN / 128; ++hh)
          if (n0 + hh * 128 < a.N) epi_qkv_head(ep, a, taddr + (uint32_t)(hh * 128), m, n0 + hh * 128);
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(taddr + (uint32_t)c, r);
          ptx::tmem_ld_wait();
          if (ep.mode == EPI_RESID || ep.mode == EPI_BLOCK_END)
            epi_resid_chunk(ep, a, epi_stage + (warp - 2) * Cf::STAGE_FLOATS, mb * kBM + g * 32, n0 + c, r,
                            lane);
          else
            epi_chunk(ep, a, m, n0 + c, r, ce_sum, ce_tgt, y);
        }
      }
      if (ep.mode == EPI_CE && m < a.M) {
        ep.ce_sum[(size_t)m * ep.ce_tiles + nb] = ce_sum;
        if (y >= n0 && y < n0 + BN) ep.ce_tgt[m] = ce_tgt;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(tempty(acc));
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Cf::TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <int BN>
void set_smem_attr() {
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(k_gemm_tc<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<BN>::SMEM);
  });
}

}  // namespace

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with row pitch
// `ld` elements; box = box_cols x box_rows, 128-byte swizzle, zero fill.
bool make_tmap_2d(CUtensorMap* map, const void* ptr, int rows, int cols, int ld, int box_rows,
                  int box_cols) {
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D bf16 tensor map over [d3][d2][d1][d0] with strides (bytes) s1, s2, s3.
bool make_tmap_4d(CUtensorMap* map, const void* ptr, const uint64_t (&dims)[4],
                  const uint64_t (&strides_bytes)[3], const uint32_t (&box)[4]) {
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return false;
  const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  const cuuint64_t s[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  const cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), d, s, b, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemm_tc_bn(int N) { return (N % 256 == 0) ? 256 : 128; }

bool launch_gemm_tc(const bf16* A, int lda, const bf16* Bm, int ldb, int M, int N, int K,
                    const EpiParams& ep, int* status, int num_sms, cudaStream_t st) {
  const int BN = gemm_tc_bn(N);
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, M, K, lda, kBM, kBK)) return false;
  if (!make_tmap_2d(&tb, Bm, N, K, ldb, BN, kBK)) return false;
  TcArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = (M + kBM - 1) / kBM;
  a.tiles_n = (N + BN - 1) / BN;
  a.num_tiles = a.tiles_m * a.tiles_n;
  a.status = status;
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  LaunchScope scope_(KK_GEMM_TC, st);
  if (BN == 256) {
    set_smem_attr<256>();
    k_gemm_tc<256><<<grid, 192, TcCfg<256>::SMEM, st>>>(ta, tb, a, ep);
  } else {
    set_smem_attr<128>();
    k_gemm_tc<128><<<grid, 192, TcCfg<128>::SMEM, st>>>(ta, tb, a, ep);
  }
  return true;
}

}  // namespace nc
