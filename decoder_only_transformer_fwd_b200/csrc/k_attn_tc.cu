// tcgen05 flash attention for sm_100a: causal sliding-window softmax
// attention, head dim 128, bf16 q/k/v, fp32 scores and accumulation.
//
// "The Mathematics of Karpathy's nanochat", §Scaled Dot-Product Attention
// with Sliding Window: query i sees key j iff j <= i and i - j < w;
// o_i = sum_j softmax_j(scale q_i . k_j) v_j.
//
// Persistent: one CTA per SM walks work items (one 128-query tile of one
// head each), heaviest first (the last query tiles see the most keys).
//   warp 0      TMA: the item's Q tile, then its K and V tiles (128 keys) into
//               a two-stage ring that runs on across items; only key tiles
//               that hold a visible key are visited, so masked work is
//               skipped tile by tile;
//   warp 1      TMEM allocation (512 columns: S0 | S1 | O0 | O1) and one
//               thread issuing tcgen05.mma: S_j = Q K_j^T (M = N = 128, K = 16
//               steps over D), then O += P_j V_j with V read as an MN-major
//               operand straight from the TMA tile;
//   warps 2..5  online softmax, one query row per thread (its TMEM lane):
//               row max on the raw scores, p = 2^(s c - m c) with the scale c
//               folded into one FMA, P_j to shared memory as bf16 in the
//               128-byte-swizzled K-major layout the MMA reads; the running
//               max moves (and O is rescaled through TMEM) only when it grows
//               by more than 2^8, so p <= 256; finally O / l to global memory.
// S_{j+1} is computed while the softmax works on S_j, and the two O buffers
// let the output of item i drain while the MMAs of item i + 1 run.  All
// barrier phases are counted over the CTA's whole sequence of tiles.  Every
// wait is bounded; on a timeout the CTA records NC_ERR_TIMEOUT and returns
// after its copies and MMAs have landed.
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
constexpr uint32_t TMEM_COLS = 512;  // S0 | S1 | O0 | O1
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnArgs {
  int B, T, H, Hkv, window;
  int ldo;
  int n_qblocks, n_items;
  float scale_log2;  // softmax_scale * log2(e)
  bf16* o;
  int* status;
};

struct Item {
  int b, h, q0, kt_lo, n_tiles;
};

// item i: query tile n_qblocks - 1 - i / (B H) (heaviest first), head-batch i % (B H)
__device__ __forceinline__ Item decode_item(const AttnArgs& a, int i) {
  Item it;
  const int bh = a.B * a.H;
  const int qb = a.n_qblocks - 1 - i / bh;
  const int r = i % bh;
  it.b = r / a.H;
  it.h = r % a.H;
  it.q0 = qb * kQ;
  it.kt_lo = max(0, it.q0 - a.window + 1) / kK;
  const int kt_hi = min(it.q0 + kQ - 1, a.T - 1) / kK;
  it.n_tiles = kt_hi - it.kt_lo + 1;
  return it;
}

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
  enum {
    B_QF = 0, B_QE = 1, B_KF = 2, B_VF = 4, B_KE = 6, B_VE = 8, B_SF = 10, B_PF = 12, B_PV = 13,
    B_OE = 14, B_DONE = 16, NB = 17
  };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(B_QF), 1);
    ptx::mbar_init(bar(B_QE), 1);
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(bar(B_KF + s), 1);
      ptx::mbar_init(bar(B_VF + s), 1);
      ptx::mbar_init(bar(B_KE + s), 1);
      ptx::mbar_init(bar(B_VE + s), 1);
      ptx::mbar_init(bar(B_SF + s), 1);
      ptx::mbar_init(bar(B_OE + s), 4);
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
      uint32_t kissued = 0, vissued = 0, kpar = 0, vpar = 0, qpar = 0;
      bool qissued = false;
      int g = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it) {
        const Item w = decode_item(a, item);
        const int row_base = w.b * a.T;
        const int qcol = w.h * kD, kcol = (w.h / (a.H / a.Hkv)) * kD;
        // the previous item's QK MMAs have finished reading the Q buffer
        if (*abort_flag || !ptx::mbar_wait(bar(B_QE), (it & 1) ^ 1, a.status)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(bar(B_QF), TILE_BYTES);
        ptx::tma_load_2d(sQ, &tmQ, bar(B_QF), qcol, row_base + w.q0);
        ptx::tma_load_2d(sQ + BOX_BYTES, &tmQ, bar(B_QF), qcol + 64, row_base + w.q0);
        qissued = true;
        qpar = it & 1;
        for (int j = 0; j < w.n_tiles; ++j, ++g) {
          const int s = g & 1;
          const uint32_t ph = (g >> 1) & 1;
          const int krow = row_base + (w.kt_lo + j) * kK;
          if (*abort_flag || !ptx::mbar_wait(bar(B_KE + s), ph ^ 1, a.status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(bar(B_KF + s), TILE_BYTES);
          ptx::tma_load_2d(sK(s), &tmK, bar(B_KF + s), kcol, krow);
          ptx::tma_load_2d(sK(s) + BOX_BYTES, &tmK, bar(B_KF + s), kcol + 64, krow);
          kissued |= 1u << s;
          kpar = (kpar & ~(1u << s)) | (ph << s);
          if (*abort_flag || !ptx::mbar_wait(bar(B_VE + s), ph ^ 1, a.status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(bar(B_VF + s), TILE_BYTES);
          ptx::tma_load_2d(sV(s), &tmV, bar(B_VF + s), kcol, krow);
          ptx::tma_load_2d(sV(s) + BOX_BYTES, &tmV, bar(B_VF + s), kcol + 64, krow);
          vissued |= 1u << s;
          vpar = (vpar & ~(1u << s)) | (ph << s);
        }
      }
      if (!ok) *abort_flag = 1;
      // every copy this thread issued has landed before the CTA may exit
      if (qissued) ptx::mbar_wait(bar(B_QF), qpar, a.status);
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
      auto issue_qk = [&](int gj) -> bool {
        const int s = gj & 1;
        if (*abort_flag || !ptx::mbar_wait(bar(B_KF + s), (gj >> 1) & 1, a.status)) return false;
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
      bool ok = true;
      int g = 0, it = 0;
      for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it) {
        const Item w = decode_item(a, item);
        const int ob = it & 1;
        const uint32_t tO = tmem + 256 + (uint32_t)(ob * 128);
        if (*abort_flag || !ptx::mbar_wait(bar(B_QF), it & 1, a.status)) { ok = false; break; }
        ptx::tc_fence_after();
        if (!issue_qk(g)) { ok = false; break; }
        if (w.n_tiles == 1) ptx::mma_commit(bar(B_QE));
        for (int j = 0; j < w.n_tiles; ++j) {
          const int gj = g + j;
          const int s = gj & 1;
          // S_{j+1} goes to the other buffer; the softmax released it with P_{j-1}
          if (j + 1 < w.n_tiles) {
            if (!issue_qk(gj + 1)) { ok = false; break; }
            if (j + 2 == w.n_tiles) ptx::mma_commit(bar(B_QE));  // last QK of the item issued
          }
          if (*abort_flag || !ptx::mbar_wait(bar(B_PF), gj & 1, a.status) ||
              !ptx::mbar_wait(bar(B_VF + s), (gj >> 1) & 1, a.status)) { ok = false; break; }
          // the output of the item two back has been read out of this O buffer
          if (j == 0 && !ptx::mbar_wait(bar(B_OE + ob), ((it >> 1) & 1) ^ 1, a.status)) { ok = false; break; }
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
        g += w.n_tiles;
      }
      if (!ok) *abort_flag = 1;
      ptx::mma_commit(bar(B_DONE));
      ptx::mbar_wait(bar(B_DONE), 0, a.status);
    }
  } else {
    // ---------------- softmax + epilogue (warps 2..5) ----------------
    const int gq = warp & 3;
    const int r = gq * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(gq * 32) << 16;
    const float c = a.scale_log2;
    bool ok = true;
    int g = 0, it = 0;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it) {
      const Item w = decode_item(a, item);
      const int qi = w.q0 + r;  // query position
      const int ob = it & 1;
      const uint32_t tO = tmem + 256 + (uint32_t)(ob * 128) + lane_off;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < w.n_tiles; ++j) {
        const int gj = g + j;
        const int s = gj & 1;
        const int k0 = (w.kt_lo + j) * kK;
        if (*abort_flag || !ptx::mbar_wait(bar(B_SF + s), (gj >> 1) & 1, a.status)) { ok = false; break; }
        ptx::tc_fence_after();
        float x[128];
        const uint32_t tS = tmem + (uint32_t)(s * 128) + lane_off;
        {
          // four TMEM loads in flight behind one wait
          uint32_t u0[32], u1[32], u2[32], u3[32];
          ptx::tmem_ld32(tS, u0);
          ptx::tmem_ld32(tS + 32, u1);
          ptx::tmem_ld32(tS + 64, u2);
          ptx::tmem_ld32(tS + 96, u3);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            x[i] = __uint_as_float(u0[i]);
            x[32 + i] = __uint_as_float(u1[i]);
            x[64 + i] = __uint_as_float(u2[i]);
            x[96 + i] = __uint_as_float(u3[i]);
          }
        }
        // visible keys of this row in this tile: columns [clo, chi]
        const int clo = qi - a.window + 1 - k0;
        const int chi = qi - k0;
        if (!(clo <= 0 && chi >= kK - 1)) {
#pragma unroll
          for (int i = 0; i < 128; ++i) x[i] = (i >= clo && i <= chi) ? x[i] : -INFINITY;
        }
        // row max as a tree (short dependency chains: one softmax warp per scheduler)
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = x[k];
#pragma unroll
        for (int i = 8; i < 128; i += 8)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], x[i + k]);
        const float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        // lazy max (raw score units): move it only when it grows by more than 2^8 after scaling
        const bool rescale = (tmax - m_run) * c > kRescaleThreshold;
        const float m_new = rescale ? tmax : m_run;
        const float mc = (m_new == -INFINITY) ? 0.f : m_new * c;
        float sm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float p0 = ex2(fmaf(x[2 * i], c, -mc)), p1 = ex2(fmaf(x[2 * i + 1], c, -mc));
          sm[i & 7] += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
        const float rsum = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
        // P_{gj-1} and O through PV_{gj-1} are done before P is rewritten or O rescaled
        if (gj > 0 && !ptx::mbar_wait(bar(B_PV), (gj - 1) & 1, a.status)) { ok = false; break; }
        ptx::tc_fence_after();
        const float alpha = rescale ? ex2(m_run * c - mc) : 1.f;  // 0 when m_run == -inf
        if (rescale) {
          l_run *= alpha;
          m_run = m_new;
        }
        // O is rescaled by the whole warp (tcgen05.ld/st are warp-collective);
        // rows that keep their max use alpha = 1
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t u[32];
            ptx::tmem_ld32(tO + (uint32_t)(cc * 32), u);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            ptx::tmem_st32(tO + (uint32_t)(cc * 32), u);
          }
          ptx::tmem_st_wait();
        }
        l_run += rsum;
        // P tile: row r, keys 8q..8q+7 -> box q/8, 16-byte chunk (q%8) ^ (r%8)
        uint8_t* prow = smem + OFF_P + r * 128;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int box = q >> 3, qq = q & 7;
          uint4* dst = reinterpret_cast<uint4*>(prow + box * BOX_BYTES + ((qq ^ (r & 7)) << 4));
          *dst = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_PF));
      }
      if (!ok) break;
      // output: O / l once the item's last PV has landed
      const int glast = g + w.n_tiles - 1;
      if (!ptx::mbar_wait(bar(B_PV), glast & 1, a.status)) { ok = false; break; }
      ptx::tc_fence_after();
      const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
      const bool store = qi < a.T;
      bf16* dst = a.o + (size_t)(w.b * a.T + qi) * a.ldo + w.h * kD;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t u[32];
        ptx::tmem_ld32(tO + (uint32_t)(cc * 32), u);
        ptx::tmem_ld_wait();
        if (store) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d4[q] = make_uint4(pack_bf16(__uint_as_float(u[8 * q + 0]) * inv, __uint_as_float(u[8 * q + 1]) * inv),
                               pack_bf16(__uint_as_float(u[8 * q + 2]) * inv, __uint_as_float(u[8 * q + 3]) * inv),
                               pack_bf16(__uint_as_float(u[8 * q + 4]) * inv, __uint_as_float(u[8 * q + 5]) * inv),
                               pack_bf16(__uint_as_float(u[8 * q + 6]) * inv, __uint_as_float(u[8 * q + 7]) * inv));
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_OE + ob));
      g += w.n_tiles;
    }
    if (!ok) *abort_flag = 1;
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
  const int M = B * T;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_2d(&tq, q, M, H * kD, ldq, kQ, 64)) return false;
  if (!make_tmap_2d(&tk, k, M, Hkv * kD, ldk, kK, 64)) return false;
  if (!make_tmap_2d(&tv, v, M, Hkv * kD, ldv, kK, 64)) return false;
  AttnArgs a;
  a.B = B;
  a.T = T;
  a.H = H;
  a.Hkv = Hkv;
  a.window = (window <= 0 || window > T) ? T : window;
  a.ldo = ldo;
  a.n_qblocks = (T + kQ - 1) / kQ;
  a.n_items = a.n_qblocks * B * H;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.o = o;
  a.status = status;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  LaunchScope scope_(KK_ATTN_TC, st);
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  k_attn_tc<<<grid, 192, SMEM_BYTES, st>>>(tq, tk, tv, a);
  return true;
}

}  // namespace nc
