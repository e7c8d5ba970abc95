// tcgen05 flash attention for sm_100a: causal sliding-window softmax
// attention, head dim 128, bf16 q/k/v, fp32 scores and accumulation.
//
// "The Mathematics of Karpathy's nanochat", §Scaled Dot-Product Attention
// with Sliding Window: query i sees key j iff j <= i and i - j < w;
// o_i = sum_j softmax_j(scale q_i . k_j) v_j.
//
// Persistent: one CTA per SM walks work items, heaviest first, in rounds of
// alternating direction.  An item is a pair of adjacent 128-query tiles
// (A, B) of one head, which share one stream of 128-key K/V tiles:
//   warps 0..3  softmax of tile A, one query row per thread (its TMEM lane);
//   warps 4..7  softmax of tile B;
//   warp 8      TMA: the item's two Q tiles, then K_t and V_t for every key
//               tile t that holds a key visible to A or B, into a 5-slot ring
//               (32 KB slots) that runs on across items;
//   warp 9      TMEM allocation (512 columns: S_A | S_B | O_A | O_B) and one
//               thread issuing tcgen05.mma: S_g = Q_g K_t^T (M = N = 128,
//               K = 16 steps over D) and O_g += P_g V_t, with P_g read from
//               tensor memory and V read as an MN-major operand straight from
//               the TMA tile;
//   warps 10,11 idle (they complete the TMA/MMA warpgroup, which hands its
//               registers to the softmax warpgroups).
// P_g overwrites the first 64 columns of S_g as packed bf16 (two keys per
// 32-bit column), so no shared memory holds P and the ring gets five slots.
// For each key tile the MMA warp issues, per group, PV_g(t) once P_g(t) is
// written and then S_g(t+1) = Q_g K_{t+1}^T into the same columns; the tensor
// core runs them in issue order, so S_g(t+1) never overwrites P_g(t) before
// it has been read, and "S_g(t+1) ready" also means "O_g holds PV_g(t)".  One
// group's exponentials overlap the other group's MMAs.  A group skips key
// tiles that hold no key visible to it, so masked work is skipped tile by
// tile.  Softmax: row max on the raw scores, p = 2^(s c - m c) with the scale
// c folded into one FMA; the running max moves (and O is rescaled through
// TMEM) only when it grows by more than 2^8, so p <= 256.  All barrier phases
// are counted over the CTA's whole sequence.  Every wait is bounded; on a
// timeout the CTA records NC_ERR_TIMEOUT and returns after its copies and
// MMAs have landed.
#include "nc_internal.cuh"
#include "ptx.cuh"

namespace nc {

bool make_tmap_2d(CUtensorMap* map, const void* ptr, int rows, int cols, int ld, int box_rows,
                  int box_cols);

namespace {

constexpr int kQ = 128, kK = 128, kD = 128;
constexpr int TILE_BYTES = kQ * kD * 2;    // 32 KB: a 128 x 128 bf16 tile (two 64-column boxes)
constexpr int BOX_BYTES = TILE_BYTES / 2;  // 16 KB: 128 rows x 64 columns
constexpr int SLOTS = 5;
// shared memory: Q_A | Q_B | slot[5] | barriers
constexpr int OFF_Q = 0;
constexpr int OFF_SLOT = OFF_Q + 2 * TILE_BYTES;
constexpr int OFF_BAR = OFF_SLOT + SLOTS * TILE_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;  // S_A | S_B | O_A | O_B
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// warps 0..3: softmax of tile A, 4..7: softmax of tile B, 8: TMA, 9: MMA, 10..11: idle
constexpr int kThreads = 384;
constexpr int kWarpTma = 8, kWarpMma = 9;
// registers: launched at 168 per thread (65536 / 384, rounded down to 8);
// the TMA/MMA warpgroup drops to kRegsLow and the two softmax warpgroups rise
// to kRegsHigh, 2 * 128 * kRegsHigh + 128 * kRegsLow <= 64512 = 384 * 168.
// The splits are those at which the compiler spills nothing (base attention:
// 120 / 192) or least (routing, with its second Q operand: 144 / 176).
template <bool ROUTE> constexpr int kRegsLow = ROUTE ? 144 : 120;
template <bool ROUTE> constexpr int kRegsHigh = ROUTE ? 176 : 192;
static_assert(2 * 128 * kRegsHigh<false> + 128 * kRegsLow<false> <= kThreads * 168, "register split");
static_assert(2 * 128 * kRegsHigh<true> + 128 * kRegsLow<true> <= kThreads * 168, "register split");

struct AttnArgs {
  int B, T, H, Hkv, window;
  int ldo;
  int o_v8;  // o is 32-byte aligned and ldo a multiple of 16: 32-byte stores
  int n_qblocks, n_pairs, n_items;
  float scale_log2;  // softmax_scale * log2(e)
  bf16* o;
  int* status;
};

struct Item {
  int b, h, q0;  // q0: first query of tile A; tile B starts at q0 + 128
  int has_b;
  int lo0, hi0;  // key tiles visible to tile A
  int lo1, hi1;  // key tiles visible to tile B (when has_b)
  int lo, hi;    // their union, which is contiguous
};

__device__ __forceinline__ int first_key_tile(const AttnArgs& a, int q0) { return max(0, q0 - a.window + 1) / kK; }
__device__ __forceinline__ int last_key_tile(const AttnArgs& a, int q0) { return min(q0 + kQ - 1, a.T - 1) / kK; }

// item i: query-tile pair n_pairs - 1 - i / (B H) (heaviest first), head-batch i % (B H).
// With ROUTE an item is a single query tile (tile A only): its two Q halves
// take both Q buffers.
template <bool ROUTE>
__device__ __forceinline__ Item decode_item(const AttnArgs& a, int i) {
  Item it;
  const int bh = a.B * a.H;
  const int p = a.n_pairs - 1 - i / bh;
  const int r = i % bh;
  it.b = r / a.H;
  it.h = r % a.H;
  it.q0 = (ROUTE ? 1 : 2) * p * kQ;
  it.has_b = !ROUTE && (2 * p + 1) < a.n_qblocks;
  it.lo0 = first_key_tile(a, it.q0);
  it.hi0 = last_key_tile(a, it.q0);
  it.lo1 = first_key_tile(a, it.q0 + kQ);
  it.hi1 = last_key_tile(a, it.q0 + kQ);
  it.lo = it.lo0;
  it.hi = it.has_b ? it.hi1 : it.hi0;
  return it;
}

// The k-th item of this CTA.  Rounds of gridDim.x items alternate direction
// (forward, then backward over the CTAs), so with items ordered heaviest first
// the CTA that took the heaviest item of one round takes the lightest of the
// next: per-CTA totals stay close to the mean without any atomics.
__device__ __forceinline__ int item_of(int k) {
  const int g = (int)gridDim.x, c = (int)blockIdx.x;
  return k * g + ((k & 1) ? g - 1 - c : c);
}

__device__ __forceinline__ bool active(const Item& it, int g, int t) {
  return g == 0 ? (t >= it.lo0 && t <= it.hi0) : (it.has_b && t >= it.lo1 && t <= it.hi1);
}

using ptx::ex2;

// Packed fp32 pairs (the f32x2 add / fma of this architecture).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ROUTE: the pass-2 attention of the looped model ("looped-nanochat-d24"
// card, routing loop): the logits gain a prior g q1 . k1 from the pass-1
// features, computed as one QK^T over the augmented width 256, [q2 | g q1] .
// [k2 | k1] (the card's own construction).  Q2 and the pre-scaled Q1 fill the
// two Q buffers (so an item is one query tile), and each key tile takes three
// ring slots: K2, K1, V.
template <bool ROUTE>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ1,
              const __grid_constant__ CUtensorMap tmK1, const AttnArgs a) {
  constexpr int PER_TILE = ROUTE ? 3 : 2;  // ring slots per key tile
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  enum {
    B_QF = 0, B_QE = 2, B_SLF = 4, B_SLE = B_SLF + SLOTS, B_S = B_SLE + SLOTS, B_P = B_S + 2, B_O = B_P + 2,
    B_OE = B_O + 2, B_DONE = B_OE + 2, NB = B_DONE + 1
  };
  static_assert(NB * 8 + 8 <= 256, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      ptx::mbar_init(bar(B_QF + g), 1);
      ptx::mbar_init(bar(B_QE + g), 1);
    }
    for (int s = 0; s < SLOTS; ++s) {
      ptx::mbar_init(bar(B_SLF + s), 1);
      ptx::mbar_init(bar(B_SLE + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      ptx::mbar_init(bar(B_S + g), 1);
      ptx::mbar_init(bar(B_P + g), 4);
      ptx::mbar_init(bar(B_O + g), 1);
      ptx::mbar_init(bar(B_OE + g), 4);
    }
    ptx::mbar_init(bar(B_DONE), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    if (ROUTE) {
      ptx::prefetch_tmap(&tmQ1);
      ptx::prefetch_tmap(&tmK1);
    }
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // q, k, v come from the previous kernel; o may still be read by it
  auto sQ = [&](int g) { return ptx::smem_u32(smem + OFF_Q + g * TILE_BYTES); };
  auto sSlot = [&](int s) { return ptx::smem_u32(smem + OFF_SLOT + s * TILE_BYTES); };

  if (warp >= 8) {
    ptx::setmaxnreg_dec<kRegsLow<ROUTE>>();
    if (warp == kWarpTma) {
    if (ptx::elect_one()) {
      // ---------------- TMA producer ----------------
      uint32_t issued = 0, par = 0;
      int qn[2] = {0, 0}, qpar[2] = {0, 0};  // Q loads issued per buffer group, parity of the last
      bool ok = true;
      int sc = 0, it = 0;
      for (int item = item_of(0); ok && item < a.n_items; ++it, item = item_of(it)) {
        const Item w = decode_item<ROUTE>(a, item);
        const int row_base = w.b * a.T;
        const int qcol = w.h * kD, kcol = (w.h / (a.H / a.Hkv)) * kD;
        // K_t (ROUTE: K2_t, K1_t) then V_t into the next ring slots
        auto load_kv = [&](int t) -> bool {
          const int krow = row_base + t * kK;
          for (int kv = 0; kv < PER_TILE; ++kv, ++sc) {
            const int s = sc % SLOTS;
            const uint32_t ph = (uint32_t)(sc / SLOTS) & 1u;
            if (*abort_flag || !ptx::mbar_wait(bar(B_SLE + s), ph ^ 1, a.status)) return false;
            const void* tm = kv == 0 ? (const void*)&tmK
                                     : (kv == PER_TILE - 1 ? (const void*)&tmV : (const void*)&tmK1);
            ptx::mbar_arrive_expect_tx(bar(B_SLF + s), TILE_BYTES);
            ptx::tma_load_2d(sSlot(s), tm, bar(B_SLF + s), kcol, krow);
            ptx::tma_load_2d(sSlot(s) + BOX_BYTES, tm, bar(B_SLF + s), kcol + 64, krow);
            issued |= 1u << s;
            par = (par & ~(1u << s)) | (ph << s);
          }
          return true;
        };
        // the item's first K/V tiles do not need the Q buffers: start them first
        if (!load_kv(w.lo)) { ok = false; break; }
        // each group's Q buffer is reloaded once that group's QK MMAs of its
        // previous item have finished reading it (ROUTE: group 0 owns both
        // buffers, Q2 in the first and the pre-scaled Q1 in the second)
        for (int g = 0; g < (ROUTE ? 1 : (w.has_b ? 2 : 1)); ++g) {
          if (*abort_flag || !ptx::mbar_wait(bar(B_QE + g), (qn[g] & 1) ^ 1, a.status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(bar(B_QF + g), (ROUTE ? 2 : 1) * TILE_BYTES);
          for (int h = 0; h < (ROUTE ? 2 : 1); ++h) {
            const int buf = ROUTE ? h : g;
            const void* tq = (ROUTE && h == 1) ? (const void*)&tmQ1 : (const void*)&tmQ;
            const int qrow = row_base + w.q0 + (ROUTE ? 0 : g * kQ);
            ptx::tma_load_2d(sQ(buf), tq, bar(B_QF + g), qcol, qrow);
            ptx::tma_load_2d(sQ(buf) + BOX_BYTES, tq, bar(B_QF + g), qcol + 64, qrow);
          }
          qpar[g] = qn[g] & 1;
          ++qn[g];
        }
        if (!ok) break;
        for (int t = w.lo + 1; ok && t <= w.hi; ++t)
          if (!load_kv(t)) ok = false;
      }
      if (!ok) *abort_flag = 1;
      // every copy this thread issued has landed before the CTA may exit
      for (int g = 0; g < 2; ++g)
        if (qn[g] > 0) ptx::mbar_wait(bar(B_QF + g), qpar[g], a.status);
      for (int s = 0; s < SLOTS; ++s)
        if (issued & (1u << s)) ptx::mbar_wait(bar(B_SLF + s), (par >> s) & 1, a.status);
    }
  } else if (warp == kWarpMma) {
    if (ptx::elect_one()) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc_qk = ptx::idesc_bf16(kQ, kK, 0, 0);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16(kQ, kD, 0, 1);  // V is MN-major
      // shared-memory descriptors are built once; the k-steps add constants
      // to their start-address field (16-byte units): K-major steps of 16
      // elements are 32 B within a 64-column box and BOX_BYTES between the
      // two boxes; the MN-major V steps are 16 rows = 2048 B
      const uint64_t dq0 = ptx::desc_kmajor_sw128(sQ(0)), dq1 = ptx::desc_kmajor_sw128(sQ(1));
      const uint64_t dk0 = ptx::desc_kmajor_sw128(sSlot(0)), dv0 = ptx::desc_mnmajor_sw128(sSlot(0), BOX_BYTES);
      auto slot_off = [&](int sc) { return (uint64_t)((sc % SLOTS) * (TILE_BYTES >> 4)); };
      // S_g = Q_g K^T; with ROUTE (group 0 only) S = Q2 K2^T + (g Q1) K1^T, the
      // second half of the 256-wide contraction continuing the same accumulation
      auto qk = [&](int g, int sc) {
        const uint32_t tS = tmem + (uint32_t)(g * 128);
#pragma unroll
        for (int half = 0; half < (ROUTE ? 2 : 1); ++half) {
          const uint64_t dq = (g == 0 && half == 0) ? dq0 : dq1, dk = dk0 + slot_off(sc + half);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t off = (uint64_t)((kk >> 2) * (BOX_BYTES >> 4) + (kk & 3) * 2);
            ptx::mma_bf16_ss(tS, dq + off, dk + off, idesc_qk, (half > 0 || kk > 0) ? 1u : 0u);
          }
        }
      };
      auto pv = [&](int g, int sc, bool first) {
        const uint32_t tP = tmem + (uint32_t)(g * 128);  // P_g: packed bf16 over the first 64 columns of S_g
        const uint32_t tO = tmem + 256 + (uint32_t)(g * 128);
        const uint64_t dv = dv0 + slot_off(sc);
#pragma unroll
        for (int kk = 0; kk < kK / 16; ++kk)
          ptx::mma_bf16_ts(tO, tP + (uint32_t)(kk * 8), dv + (uint64_t)(kk * (2048 >> 4)), idesc_pv,
                           (!first || kk > 0) ? 1u : 0u);
      };
      auto slot_wait = [&](int sc) -> bool {
        return !*abort_flag && ptx::mbar_wait(bar(B_SLF + sc % SLOTS), (uint32_t)(sc / SLOTS) & 1u, a.status);
      };
      // group g's Q buffer holds the current item's tile (QF_g phase qc[g])
      int qc[2] = {0, 0};
      auto q_wait = [&](int g) -> bool {
        const bool r = !*abort_flag && ptx::mbar_wait(bar(B_QF + g), qc[g] & 1, a.status);
        ++qc[g];
        return r;
      };
      bool ok = true;
      int sc = 0, it = 0;
      int pc0 = 0, pc1 = 0, ic0 = 0, ic1 = 0;  // P phases consumed, items finished, per group
      bool a_started = false;  // tile A's first QK of this item was issued during the previous item
      for (int item = item_of(0); ok && item < a.n_items; ++it, item = item_of(it)) {
        const Item w = decode_item<ROUTE>(a, item);
        // K_lo feeds the first S of every group that sees key tile lo
        if (!slot_wait(sc) || (ROUTE && !slot_wait(sc + 1))) { ok = false; break; }
#pragma unroll
        for (int g = 0; g < 2; ++g)
          if (active(w, g, w.lo) && !(g == 0 && a_started)) {
            if (!q_wait(g)) { ok = false; break; }
            ptx::tc_fence_after();
            qk(g, sc);
            ptx::mma_commit(bar(B_S + g));
            if (w.lo == (g == 0 ? w.hi0 : w.hi1)) ptx::mma_commit(bar(B_QE + g));  // g's only tile
          }
        if (!ok) break;
        a_started = false;
        ptx::mma_commit(bar(B_SLE + sc % SLOTS));
        if (ROUTE) ptx::mma_commit(bar(B_SLE + (sc + 1) % SLOTS));
        for (int t = w.lo; ok && t <= w.hi; ++t) {
          const int scV = sc + PER_TILE * (t - w.lo) + PER_TILE - 1, scK1 = scV + 1;
          const bool more = t < w.hi;
          if (!slot_wait(scV) || (more && !slot_wait(scK1)) || (ROUTE && more && !slot_wait(scK1 + 1))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const bool act = active(w, g, t);
            const bool next = more && active(w, g, t + 1);
            if (act) {
              // group g has written P_g(t)
              int& pc = g == 0 ? pc0 : pc1;
              if (*abort_flag || !ptx::mbar_wait(bar(B_P + g), pc & 1, a.status)) { ok = false; break; }
              ++pc;
              const bool first = t == (g == 0 ? w.lo0 : w.lo1);
              // the output of this group's previous item has been read out of O_g
              const int ic = g == 0 ? ic0 : ic1;
              if (first && !ptx::mbar_wait(bar(B_OE + g), (ic & 1) ^ 1, a.status)) { ok = false; break; }
              ptx::tc_fence_after();
              pv(g, scV, first);
            }
            if (next) {
              // tile B's first key tile may follow the item's first (its Q was not needed before)
              if (!act && !q_wait(g)) { ok = false; break; }
              ptx::tc_fence_after();
              qk(g, scK1);
              ptx::mma_commit(bar(B_S + g));
              if (t + 1 == (g == 0 ? w.hi0 : w.hi1)) ptx::mma_commit(bar(B_QE + g));  // g's last QK of the item
            } else if (act) {
              ptx::mma_commit(bar(B_O + g));  // g's last tile of this item: O_g is final
              const int nitem = item_of(it + 1);
              if (g == 0 && nitem < a.n_items) {
                // tile A is done with this item: start its next item's first S
                // now, while tile B still works on its last key tiles
                const Item wn = decode_item<ROUTE>(a, nitem);
                const int scn = sc + PER_TILE * (w.hi - w.lo + 1);
                if (!q_wait(0) || !slot_wait(scn) || (ROUTE && !slot_wait(scn + 1))) { ok = false; break; }
                ptx::tc_fence_after();
                qk(0, scn);
                ptx::mma_commit(bar(B_S + 0));
                if (wn.lo0 == wn.hi0) ptx::mma_commit(bar(B_QE + 0));
                a_started = true;
              }
            }
          }
          if (!ok) break;
          ptx::mma_commit(bar(B_SLE + scV % SLOTS));
          if (more) ptx::mma_commit(bar(B_SLE + scK1 % SLOTS));
          if (ROUTE && more) ptx::mma_commit(bar(B_SLE + (scK1 + 1) % SLOTS));
        }
        ++ic0;
        if (w.has_b) ++ic1;
        sc += PER_TILE * (w.hi - w.lo + 1);
      }
      if (!ok) *abort_flag = 1;
      ptx::mma_commit(bar(B_DONE));
      ptx::mbar_wait(bar(B_DONE), 0, a.status);
    }
    }
  } else {
    ptx::setmaxnreg_inc<kRegsHigh<ROUTE>>();
    // ---------------- softmax + epilogue: group 0 = warps 0..3, group 1 = warps 4..7 ----------------
    const int g = warp >> 2;
    const int gq = warp & 3;
    const int r = gq * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(gq * 32) << 16;
    const uint32_t tS = tmem + (uint32_t)(g * 128) + lane_off;
    const uint32_t tO = tmem + 256 + (uint32_t)(g * 128) + lane_off;
    const float c = a.scale_log2;
    bool ok = true;
    int cnt = 0, icnt = 0;
    for (int k = 0, item = item_of(0); ok && item < a.n_items; ++k, item = item_of(k)) {
      const Item w = decode_item<ROUTE>(a, item);
      if (g == 1 && !w.has_b) continue;
      const int qg = w.q0 + g * kQ;  // first query of this group's tile
      const int qi = qg + r;         // query position
      const int t_lo = first_key_tile(a, qg);
      const int t_hi = last_key_tile(a, qg);
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = t_lo; t <= t_hi; ++t) {
        const int k0 = t * kK;
        // S_g(t) is ready, and O_g holds every PV of this group issued before it
        if (*abort_flag || !ptx::mbar_wait(bar(B_S + g), cnt & 1, a.status)) { ok = false; break; }
        ptx::tc_fence_after();
        float x[128];
        // visible keys of this row in this tile: columns [clo, chi]
        const int clo = qi - a.window + 1 - k0;
        const int chi = qi - k0;
        const bool full_tile = clo <= 0 && chi >= kK - 1;
        float2 sm[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 c2 = make_float2(c, c);
        // p = 2^(s c - m c) for quarter qd (32 keys), packed to bf16 over S's columns [16 qd, 16 qd + 16)
        auto exp_quarter = [&](int qd, float mcq) {
          const float2 mc2 = make_float2(-mcq, -mcq);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 e = ffma2(make_float2(x[32 * qd + 2 * i], x[32 * qd + 2 * i + 1]), c2, mc2);
            const float2 p = make_float2(ex2(e.x), ex2(e.y));
            sm[i & 3] = fadd2(sm[i & 3], p);
            pk[i] = pack_bf16(p.x, p.y);
          }
          ptx::tmem_st16(tS + (uint32_t)(16 * qd), pk);
        };
        float mx[8];
        bool rescale;
        float mc, m_new;
        // four TMEM loads in flight behind one wait; the row max first
        {
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
        // A warp whose 32 rows see every key of the tile takes the plain path.
        // Otherwise masking is decided per 32-key quarter for the whole warp
        // (its rows' visible ranges are consecutive): a quarter that every row
        // sees needs no select, one that no row sees gets P = 0 without its
        // exponentials, and only the quarters between take per-key selects.
        const bool warp_full = __all_sync(0xffffffffu, full_tile);
        unsigned vis = 0xFu;  // bit qd: some row sees quarter qd
        if (warp_full) {
          // row max: eight chains of three-input max
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmaxf(x[2 * k], x[2 * k + 1]);
#pragma unroll
          for (int i = 16; i < 128; i += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], x[i + 2 * k], x[i + 2 * k + 1]);
        } else {
          const int lo_min = __reduce_min_sync(0xffffffffu, clo), lo_max = __reduce_max_sync(0xffffffffu, clo);
          const int hi_min = __reduce_min_sync(0xffffffffu, chi), hi_max = __reduce_max_sync(0xffffffffu, chi);
          vis = 0u;
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            const int b0 = 32 * qd, b1 = 32 * qd + 31;
            if (b1 < lo_min || b0 > hi_max) continue;  // no row sees this quarter
            vis |= 1u << qd;
            if (!(b0 >= lo_max && b1 <= hi_min)) {     // some row sees only part of it
#pragma unroll
              for (int i = 32 * qd; i < 32 * qd + 32; ++i) x[i] = (i >= clo && i <= chi) ? x[i] : -INFINITY;
            }
#pragma unroll
            for (int i = 32 * qd; i < 32 * qd + 32; i += 16)
#pragma unroll
              for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], x[i + 2 * k], x[i + 2 * k + 1]);
          }
        }
        const float tmax = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        // lazy max (raw score units): move it only when it grows by more than 2^8 after scaling
        rescale = (tmax - m_run) * c > kRescaleThreshold;
        m_new = rescale ? tmax : m_run;
        mc = (m_new == -INFINITY) ? 0.f : m_new * c;
        if (warp_full) {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) exp_quarter(qd, mc);
        } else {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            if (vis & (1u << qd)) {
              exp_quarter(qd, mc);
            } else {
              uint32_t z[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) z[i] = 0u;
              ptx::tmem_st16(tS + (uint32_t)(16 * qd), z);
            }
          }
        }
        const float alpha = rescale ? ex2(m_run * c - mc) : 1.f;  // 0 when m_run == -inf
        if (rescale) {
          l_run *= alpha;
          m_run = m_new;
        }
        // O (which holds every earlier PV of this group) is rescaled by the
        // whole warp, as tcgen05.ld/st are warp-collective; rows that keep
        // their max use alpha = 1
        if (t != t_lo && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t u[32];
            ptx::tmem_ld32(tO + (uint32_t)(cc * 32), u);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            ptx::tmem_st32(tO + (uint32_t)(cc * 32), u);
          }
        }
        const float2 s01 = fadd2(sm[0], sm[1]), s23 = fadd2(sm[2], sm[3]);
        const float2 s4 = fadd2(s01, s23);
        l_run += s4.x + s4.y;
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_P + g));
        ++cnt;
      }
      if (!ok) break;
      // output: O / l once the group's last PV of the item has landed
      if (!ptx::mbar_wait(bar(B_O + g), icnt & 1, a.status)) { ok = false; break; }
      ++icnt;
      ptx::tc_fence_after();
      const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
      // O_g is read one 32-column chunk at a time and stored; it is released
      // to the next item's P V as soon as its last chunk is in registers
      uint4* d4 = reinterpret_cast<uint4*>(a.o + (size_t)(w.b * a.T + qi) * a.ldo + w.h * kD);
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t u[32];
        ptx::tmem_ld32(tO + (uint32_t)(cc * 32), u);
        ptx::tmem_ld_wait();
        if (cc == 3) {
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bar(B_OE + g));
        }
        if (qi < a.T) {
          // each thread writes its own row: whole 32-byte sectors when the
          // layout allows, else 16-byte halves
          if (a.o_v8) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t wv[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                wv[e] = pack_bf16(__uint_as_float(u[16 * hh + 2 * e]) * inv, __uint_as_float(u[16 * hh + 2 * e + 1]) * inv);
              ptx::st_global_v8(d4 + 4 * cc + 2 * hh, wv);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              d4[4 * cc + q] = make_uint4(pack_bf16(__uint_as_float(u[8 * q + 0]) * inv, __uint_as_float(u[8 * q + 1]) * inv),
                                          pack_bf16(__uint_as_float(u[8 * q + 2]) * inv, __uint_as_float(u[8 * q + 3]) * inv),
                                          pack_bf16(__uint_as_float(u[8 * q + 4]) * inv, __uint_as_float(u[8 * q + 5]) * inv),
                                          pack_bf16(__uint_as_float(u[8 * q + 6]) * inv, __uint_as_float(u[8 * q + 7]) * inv));
          }
        }
      }
    }
    if (!ok) *abort_flag = 1;
  }
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

namespace {

bool launch_attn_common(const bf16* q, const bf16* k, const bf16* v, const bf16* q1, const bf16* k1, int ldq,
                        int ldk, int ldv, bf16* o, int ldo, int B, int T, int H, int Hkv, int window, float scale,
                        int* status, int num_sms, cudaStream_t st) {
  const bool route = q1 != nullptr;
  const int M = B * T;
  CUtensorMap tq, tk, tv, tq1, tk1;
  if (!make_tmap_2d(&tq, q, M, H * kD, ldq, kQ, 64)) return false;
  if (!make_tmap_2d(&tk, k, M, Hkv * kD, ldk, kK, 64)) return false;
  if (!make_tmap_2d(&tv, v, M, Hkv * kD, ldv, kK, 64)) return false;
  if (!make_tmap_2d(&tq1, route ? q1 : q, M, H * kD, ldq, kQ, 64)) return false;
  if (!make_tmap_2d(&tk1, route ? k1 : k, M, Hkv * kD, ldk, kK, 64)) return false;
  AttnArgs a;
  a.B = B;
  a.T = T;
  a.H = H;
  a.Hkv = Hkv;
  a.window = (window <= 0 || window > T) ? T : window;
  a.ldo = ldo;
  a.o_v8 = (reinterpret_cast<uintptr_t>(o) % 32 == 0) && (ldo % 16 == 0);
  a.n_qblocks = (T + kQ - 1) / kQ;
  a.n_pairs = route ? a.n_qblocks : (a.n_qblocks + 1) / 2;
  a.n_items = a.n_pairs * B * H;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.o = o;
  a.status = status;
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, AttnArgs) =
      route ? k_attn_tc<true> : k_attn_tc<false>;
  if (!smem_optin(kern, SMEM_BYTES)) return false;
  LaunchScope scope_(KK_ATTN_TC, st);
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), SMEM_BYTES, st, 1, tq, tk, tv, tq1, tk1, a) == cudaSuccess;
}

}  // namespace

bool launch_attn_tc(const bf16* q, const bf16* k, const bf16* v, int ldq, int ldk, int ldv, bf16* o,
                    int ldo, int B, int T, int H, int Hkv, int window, float scale, int* status,
                    int num_sms, cudaStream_t st) {
  return launch_attn_common(q, k, v, nullptr, nullptr, ldq, ldk, ldv, o, ldo, B, T, H, Hkv, window, scale, status,
                            num_sms, st);
}

bool launch_attn_route_tc(const bf16* q2, const bf16* k2, const bf16* v2, const bf16* q1s, const bf16* k1, bf16* o,
                          int B, int T, int H, int Hkv, int window, float scale, int* status, int num_sms,
                          cudaStream_t st) {
  return launch_attn_common(q2, k2, v2, q1s, k1, H * kD, Hkv * kD, Hkv * kD, o, H * kD, B, T, H, Hkv, window, scale,
                            status, num_sms, st);
}

}  // namespace nc
