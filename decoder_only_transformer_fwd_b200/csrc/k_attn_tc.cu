// tcgen05 flash attention for sm_100a: causal sliding-window softmax
// attention, head dim 128, bf16 q/k/v, fp32 scores and accumulation.
//
// "The Mathematics of Karpathy's nanochat", §Scaled Dot-Product Attention
// with Sliding Window: query i sees key j iff j <= i and i - j < w;
// o_i = sum_j softmax_j(scale q_i . k_j) v_j.
//
// One CTA computes one 128-query tile of one head:
//   warp 0      TMA: the Q tile once, then K and V tiles (128 keys) into a
//               two-stage ring; only the key tiles that hold a visible key
//               are visited, so masked work is skipped tile by tile;
//   warp 1      TMEM allocation (512 columns: two S buffers and O) and one
//               thread issuing tcgen05.mma: S_j = Q K_j^T (M = N = 128,
//               K = 16 steps over D), then O += P_j V_j with V read as an
//               MN-major operand straight from the TMA tile;
//   warps 2..5  online softmax, one query row per thread (its TMEM lane):
//               row max, exp2, row sum, P_j to shared memory as bf16 in the
//               128-byte-swizzled K-major layout the MMA reads; the running
//               max is only moved (and O rescaled through TMEM) when it
//               grows by more than 2^8, so p <= 256 and no rescale is needed
//               in the common case; finally O / l to global memory.
// S_{j+1} is computed while the softmax works on S_j.  Every wait is
// bounded; on a timeout the CTA records NC_ERR_TIMEOUT and returns after its
// copies and MMAs have landed.
#include <mutex>

#include "nc_internal.cuh"
#include "ptx.cuh"

namespace nc {

bool make_tmap_2d(CUtensorMap* map, const void* ptr, int rows, int cols, int ld, int box_rows,
                  int box_cols);

namespace {

constexpr int kQ = 128, kK = 128, kD = 128;
constexpr int TILE_BYTES = kQ * kD * 2;   // 32 KB: a 128 x 128 bf16 tile (two 64-column boxes)
constexpr int BOX_BYTES = TILE_BYTES / 2; // 16 KB: 128 rows x 64 columns
constexpr int STAGES = 2;
// shared memory: Q | K[2] | V[2] | P | barriers
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;
constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
constexpr int OFF_P = OFF_V + STAGES * TILE_BYTES;
constexpr int OFF_BAR = OFF_P + TILE_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;  // S0 | S1 | O | (unused)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnArgs {
  int T, H, Hkv, window;
  int ldo;
  int n_qblocks;
  float scale_log2;  // softmax_scale * log2(e)
  bf16* o;
  int* status;
};

using ptx::ex2;

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(192, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  // barriers
  enum { B_Q = 0, B_KF = 1, B_VF = 3, B_KE = 5, B_VE = 7, B_SF = 9, B_PF = 11, B_PV = 12, B_DONE = 13, NB = 14 };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // heavy tiles first: the last query tiles see the most keys
  const int qb = a.n_qblocks - 1 - (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (a.H / a.Hkv);
  const int q0 = qb * kQ;
  const int kt_lo = max(0, q0 - a.window + 1) / kK;
  const int kt_hi = min(q0 + kQ - 1, a.T - 1) / kK;
  const int n_tiles = kt_hi - kt_lo + 1;
  const int row_base = b * a.T;  // first row of this sequence in the [B*T, ld] views

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(B_Q), 1);
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(bar(B_KF + s), 1);
      ptx::mbar_init(bar(B_VF + s), 1);
      ptx::mbar_init(bar(B_KE + s), 1);
      ptx::mbar_init(bar(B_VE + s), 1);
      ptx::mbar_init(bar(B_SF + s), 1);
    }
    ptx::mbar_init(bar(B_PF), 4);
    ptx::mbar_init(bar(B_PV), 1);
    ptx::mbar_init(bar(B_DONE), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sQ = ptx::smem_u32(smem + OFF_Q);
  const uint32_t sP = ptx::smem_u32(smem + OFF_P);
  auto sK = [&](int s) { return ptx::smem_u32(smem + OFF_K + s * TILE_BYTES); };
  auto sV = [&](int s) { return ptx::smem_u32(smem + OFF_V + s * TILE_BYTES); };

  if (warp == 0) {
    if (ptx::elect_one()) {
      // ---------------- TMA producer ----------------
      const int qcol = h * kD, kcol = hk * kD;
      ptx::mbar_arrive_expect_tx(bar(B_Q), TILE_BYTES);
      ptx::tma_load_2d(sQ, &tmQ, bar(B_Q), qcol, row_base + q0);
      ptx::tma_load_2d(sQ + BOX_BYTES, &tmQ, bar(B_Q), qcol + 64, row_base + q0);
      uint32_t kissued = 0, vissued = 0, kpar = 0, vpar = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int krow = row_base + (kt_lo + j) * kK;
        if (*abort_flag || !ptx::mbar_wait(bar(B_KE + s), ph ^ 1, a.status)) { *abort_flag = 1; break; }
        ptx::mbar_arrive_expect_tx(bar(B_KF + s), TILE_BYTES);
        ptx::tma_load_2d(sK(s), &tmK, bar(B_KF + s), kcol, krow);
        ptx::tma_load_2d(sK(s) + BOX_BYTES, &tmK, bar(B_KF + s), kcol + 64, krow);
        kissued |= 1u << s;
        kpar = (kpar & ~(1u << s)) | (ph << s);
        if (*abort_flag || !ptx::mbar_wait(bar(B_VE + s), ph ^ 1, a.status)) { *abort_flag = 1; break; }
        ptx::mbar_arrive_expect_tx(bar(B_VF + s), TILE_BYTES);
        ptx::tma_load_2d(sV(s), &tmV, bar(B_VF + s), kcol, krow);
        ptx::tma_load_2d(sV(s) + BOX_BYTES, &tmV, bar(B_VF + s), kcol + 64, krow);
        vissued |= 1u << s;
        vpar = (vpar & ~(1u << s)) | (ph << s);
      }
      // every copy this thread issued has landed before the CTA may exit
      ptx::mbar_wait(bar(B_Q), 0, a.status);
      for (int s = 0; s < STAGES; ++s) {
        if (kissued & (1u << s)) ptx::mbar_wait(bar(B_KF + s), (kpar >> s) & 1, a.status);
        if (vissued & (1u << s)) ptx::mbar_wait(bar(B_VF + s), (vpar >> s) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    if (ptx::elect_one()) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc_qk = ptx::idesc_bf16(kQ, kK, 0, 0);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16(kQ, kD, 0, 1);  // V is MN-major
      const uint32_t tO = tmem + 256;
      bool ok = ptx::mbar_wait(bar(B_Q), 0, a.status);
      auto issue_qk = [&](int j) -> bool {
        const int s = j & 1;
        if (*abort_flag || !ptx::mbar_wait(bar(B_KF + s), (j >> 1) & 1, a.status)) return false;
        ptx::tc_fence_after();
        const uint32_t tS = tmem + (uint32_t)(s * 128);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * BOX_BYTES + (kk & 3) * 32);
          ptx::mma_bf16_ss(tS, ptx::desc_kmajor_sw128(sQ + off), ptx::desc_kmajor_sw128(sK(s) + off),
                           idesc_qk, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(B_KE + s));
        ptx::mma_commit(bar(B_SF + s));
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j & 1;
        // S_{j+1} goes to the other buffer; the softmax released it with P_{j-1}
        if (j + 1 < n_tiles && !issue_qk(j + 1)) { ok = false; break; }
        if (*abort_flag || !ptx::mbar_wait(bar(B_PF), j & 1, a.status) ||
            !ptx::mbar_wait(bar(B_VF + s), (j >> 1) & 1, a.status)) { ok = false; break; }
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kK / 16; ++kk) {
          const uint32_t aoff = (uint32_t)((kk >> 2) * BOX_BYTES + (kk & 3) * 32);
          ptx::mma_bf16_ss(tO, ptx::desc_kmajor_sw128(sP + aoff),
                           ptx::desc_mnmajor_sw128(sV(s) + (uint32_t)(kk * 2048), BOX_BYTES), idesc_pv,
                           (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(bar(B_VE + s));
        ptx::mma_commit(bar(B_PV));
      }
      if (!ok) *abort_flag = 1;
      ptx::mma_commit(bar(B_DONE));
      ptx::mbar_wait(bar(B_DONE), 0, a.status);
    }
  } else {
    // ---------------- softmax + epilogue (warps 2..5) ----------------
    const int g = warp & 3;
    const int r = g * 32 + lane;  // row of the tile == TMEM lane
    const int qi = q0 + r;         // query position
    const uint32_t lane_off = (uint32_t)(g * 32) << 16;
    const uint32_t tO = tmem + 256 + lane_off;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      const int k0 = (kt_lo + j) * kK;
      if (*abort_flag || !ptx::mbar_wait(bar(B_SF + s), (j >> 1) & 1, a.status)) { ok = false; break; }
      ptx::tc_fence_after();
      float x[128];
      const uint32_t tS = tmem + (uint32_t)(s * 128) + lane_off;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        ptx::tmem_ld32(tS + (uint32_t)(c * 32), u);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(u[i]) * a.scale_log2;
      }
      // visible keys of this row in this tile: columns [clo, chi]
      const int clo = qi - a.window + 1 - k0;
      const int chi = qi - k0;
      const bool full = clo <= 0 && chi >= kK - 1;
      float tmax = -INFINITY;
      if (full) {
#pragma unroll
        for (int i = 0; i < 128; ++i) tmax = fmaxf(tmax, x[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          x[i] = (i >= clo && i <= chi) ? x[i] : -INFINITY;
          tmax = fmaxf(tmax, x[i]);
        }
      }
      // lazy max: move it only when it grows by more than the threshold
      const bool rescale = tmax > m_run + kRescaleThreshold;
      const float m_new = rescale ? tmax : m_run;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      float rsum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float p0 = ex2(x[2 * i] - m_use), p1 = ex2(x[2 * i + 1] - m_use);
        rsum += p0 + p1;
        pk[i] = pack_bf16(p0, p1);
      }
      // P_{j-1} and O through PV_{j-1} are done before P is rewritten or O rescaled
      if (j > 0 && !ptx::mbar_wait(bar(B_PV), (j - 1) & 1, a.status)) { ok = false; break; }
      ptx::tc_fence_after();
      const float alpha = rescale ? ex2(m_run - m_use) : 1.f;  // 0 when m_run == -inf
      if (rescale) {
        l_run *= alpha;
        m_run = m_new;
      }
      // O is rescaled by the whole warp (tcgen05.ld/st are warp-collective);
      // rows that keep their max use alpha = 1
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t u[32];
          ptx::tmem_ld32(tO + (uint32_t)(c * 32), u);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          ptx::tmem_st32(tO + (uint32_t)(c * 32), u);
        }
        ptx::tmem_st_wait();
      }
      l_run += rsum;
      // P tile: row r, keys 8c..8c+7 -> box c/8, 16-byte chunk (c%8) ^ (r%8)
      uint8_t* prow = smem + OFF_P + r * 128;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int box = c >> 3, cc = c & 7;
        uint4* dst = reinterpret_cast<uint4*>(prow + box * BOX_BYTES + ((cc ^ (r & 7)) << 4));
        *dst = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_PF));
    }
    if (ok && ptx::mbar_wait(bar(B_PV), (n_tiles - 1) & 1, a.status)) {
      ptx::tc_fence_after();
      const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
      const bool store = qi < a.T;
      bf16* dst = a.o + (size_t)(row_base + qi) * a.ldo + h * kD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        ptx::tmem_ld32(tO + (uint32_t)(c * 32), u);
        ptx::tmem_ld_wait();
        if (store) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d4[q] = make_uint4(pack_bf16(__uint_as_float(u[8 * q + 0]) * inv, __uint_as_float(u[8 * q + 1]) * inv),
                               pack_bf16(__uint_as_float(u[8 * q + 2]) * inv, __uint_as_float(u[8 * q + 3]) * inv),
                               pack_bf16(__uint_as_float(u[8 * q + 4]) * inv, __uint_as_float(u[8 * q + 5]) * inv),
                               pack_bf16(__uint_as_float(u[8 * q + 6]) * inv, __uint_as_float(u[8 * q + 7]) * inv));
        }
      }
    } else {
      *abort_flag = 1;
    }
    ptx::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

bool launch_attn_tc(const bf16* q, const bf16* k, const bf16* v, int ldq, int ldk, int ldv, bf16* o,
                    int ldo, int B, int T, int H, int Hkv, int window, float scale, int* status,
                    int num_sms, cudaStream_t st) {
  (void)num_sms;
  const int M = B * T;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_2d(&tq, q, M, H * kD, ldq, kQ, 64)) return false;
  if (!make_tmap_2d(&tk, k, M, Hkv * kD, ldk, kK, 64)) return false;
  if (!make_tmap_2d(&tv, v, M, Hkv * kD, ldv, kK, 64)) return false;
  AttnArgs a;
  a.T = T;
  a.H = H;
  a.Hkv = Hkv;
  a.window = (window <= 0 || window > T) ? T : window;
  a.ldo = ldo;
  a.n_qblocks = (T + kQ - 1) / kQ;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.o = o;
  a.status = status;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  LaunchScope scope_(KK_ATTN_TC, st);
  dim3 grid(a.n_qblocks, H, B);
  k_attn_tc<<<grid, 192, SMEM_BYTES, st>>>(tq, tk, tv, a);
  return true;
}

}  // namespace nc
