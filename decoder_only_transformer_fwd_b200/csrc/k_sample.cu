// Next-token step of generation: the softcapped logits of the last position
// of each row, then one token per row drawn from them.
//
// "The Mathematics of Karpathy's nanochat", §Inference: Generating Text: a
// forward pass gives the logits z in R^V at the last position only; §Sampling
// Controls: top-k keeps the entries z_v >= (k-th largest z), temperature tau
// divides them, P(v) = exp(z_v / tau) / sum_v' exp(z_v' / tau), one index is
// drawn from P; tau = 0 is greedy decoding (argmax).  §Logit Softcap:
// z = cap * tanh(x_L W_U^T / cap) with x_L = RMSNorm(final residual).
//
// The draw takes its uniform number u in [0, 1) from the caller: the index is
// the first v (vocabulary order) whose cumulative weight exceeds u * sum.
#include "nc_internal.cuh"
#include "ptx.cuh"

namespace nc {

bool make_tmap_2d(CUtensorMap* map, const void* ptr, int rows, int cols, int ld, int box_rows,
                  int box_cols);

namespace {

constexpr int kLastRows = 8;  // rows of one k_last_logits launch

// W_U's element type: bf16 in bf16 mode, fp32 otherwise.  A 16-byte chunk
// holds 8 or 4 elements, unpacked to fp32 pairs.  round() gives the value an
// x element takes in the product: rounded to bf16 in bf16 mode, as the head
// GEMM of the full forward rounds it (the staged copy is held as fp32).
template <typename TW> struct Chunk;
template <> struct Chunk<bf16> {
  static constexpr int kN = 8;
  __device__ static void unpack(const uint4& u, float2* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
  }
  __device__ static bf16 round(float v) { return __float2bfloat16_rn(v); }
};
template <> struct Chunk<float> {
  static constexpr int kN = 4;
  __device__ static void unpack(const uint4& u, float2* f) {
    f[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
    f[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
  __device__ static float round(float v) { return v; }
};

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// k_last_logits: warps 0..7 multiply (two groups of 4 that take alternate
// stages), warp 8 streams W_U into the ring.  Each consumer warp multiplies
// four vocabulary rows together, so every staged x value read from shared
// memory serves four rows (shared-memory traffic, not HBM, bounded the
// two-row form).
constexpr int kLastGroupWarps = 4;
constexpr int kLastConsumers = 2 * kLastGroupWarps;
constexpr int kLastThreads = 32 * (kLastConsumers + 1);
constexpr int kLastR = 4;  // vocabulary rows a consumer warp multiplies together

// The ring geometry for rows of `row_bytes`: kLastGroupWarps * kLastR rows
// per stage, 4 or 2 stages, as fit next to the staged x rows (fp32).
struct LastGeom {
  int rows, stages;
  size_t stage_bytes, x_bytes, smem;
};
inline LastGeom last_geom(int C, int esz, int nb) {
  LastGeom g;
  const size_t row_bytes = (size_t)C * esz;
  g.rows = kLastGroupWarps * kLastR;
  g.stage_bytes = (size_t)g.rows * row_bytes;
  g.x_bytes = (size_t)nb * C * 4;
  const size_t budget = 220 * 1024 - g.x_bytes - 1024;
  g.stages = (int)(budget / g.stage_bytes);
  // an even count, so that every block a stage holds belongs to the same
  // consumer group: each group then waits on consecutive phases of its stages
  g.stages = g.stages >= 4 ? 4 : (g.stages >= 2 ? 2 : 0);
  g.smem = g.stages * g.stage_bytes + g.x_bytes + 2 * 4 * 8 + 128;
  return g;
}

// Sums 2^K values across the warp at once (a transposing butterfly): on
// return, lane l holds the warp-wide total of value index
// v(l) = sum_r ((l >> (4 - r)) & 1) << (K - 1 - r), r < K.
template <int K>
__device__ __forceinline__ float warp_reduce_many(float (&a)[1 << K], int lane) {
#pragma unroll
  for (int r = 0; r < K; ++r) {
    const int bit = 4 - r, half = 1 << (K - 1 - r);
    const bool hi = (lane >> bit) & 1;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = hi ? a[i] : a[i + half];
      const float keep = hi ? a[i + half] : a[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << bit);
    }
  }
  float d = a[0];
#pragma unroll
  for (int bit = 4 - K; bit >= 0; --bit) d += __shfl_xor_sync(0xffffffffu, d, 1 << bit);
  return d;
}

// logits[b0 + j][v] = cap * tanh(rs_j * (x_j . W_U[v]) / cap) for the NB rows
// x_j = x[(b0 + j) T + T - 1], rs_j = 1 / sqrt(mean(x_j^2) + eps).  In bf16
// mode x_j is rounded to bf16 (as the head GEMM of the full forward rounds
// it) and held as fp32.  One CTA per SM; CTA c takes the blocks of `rows`
// consecutive vocabulary rows c, c + G, c + 2G, ...  One thread copies each
// block (contiguous in W_U) into a ring of shared-memory stages with a bulk
// copy; the two groups of consumer warps take alternate blocks, each warp
// multiplies four rows against the staged x rows, and the group releases the
// stage.
template <typename TW, int NB>
__global__ void __launch_bounds__(kLastThreads, 1)
k_last_logits(const float* __restrict__ x, int ldx, int T, int b0, const TW* __restrict__ W, int V, int C,
              float cap, float eps, float* __restrict__ out, int ldo, int stages, int* status) {
  pdl_launch_dependents();
  constexpr int kN = Chunk<TW>::kN;  // elements of a 16-byte chunk of W_U
  constexpr int kH = kN / 4;         // float4s of x per chunk
  constexpr int kNV = NB <= 4 ? 4 : 8;
  constexpr int kK = NB <= 4 ? 4 : 5;  // log2(kLastR * kNV)
  static_assert((1 << kK) == kLastR * kNV, "one value per (row, x row) slot");
  constexpr int rows = kLastGroupWarps * kLastR;
  extern __shared__ __align__(16) unsigned char sh_raw[];
  const size_t row_bytes = (size_t)C * sizeof(TW);
  const size_t stage_bytes = (size_t)rows * row_bytes;
  const int nchunks = C / kN;
  unsigned char* ring = sh_raw;
  // x as fp32: plane (j, h) holds float4 h of every chunk of row j, so a warp
  // reading consecutive chunks reads consecutive 16-byte words
  float4* xq = reinterpret_cast<float4*>(sh_raw + stages * stage_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sh_raw + stages * stage_bytes + (size_t)NB * C * 4);
  __shared__ float red[kLastConsumers];
  __shared__ float rs[NB];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full = [&](int s) { return ptx::smem_u32(bars + s); };
  auto empty = [&](int s) { return ptx::smem_u32(bars + 4 + s); };
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), kLastGroupWarps);
    }
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  const int nblk = (V + rows - 1) / rows;
  if (warp == kLastConsumers) {
    if (lane == 0) {
      int k = 0;
      for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, ++k) {
        const int s = k % stages;
        const uint32_t ph = (uint32_t)(k / stages) & 1u;
        if (abort_flag || !ptx::mbar_wait(empty(s), ph ^ 1u, status)) { abort_flag = 1; break; }
        const int r0 = blk * rows;
        const int nr = V - r0 < rows ? V - r0 : rows;
        const uint32_t bytes = (uint32_t)(nr * row_bytes);
        ptx::mbar_arrive_expect_tx(full(s), bytes);
        ptx::bulk_load(ptx::smem_u32(ring + s * stage_bytes), W + (size_t)r0 * C, bytes, full(s));
      }
      // every copy this thread issued has landed before the CTA may exit
      const int issued = k;
      for (int q = issued - stages > 0 ? issued - stages : 0; q < issued; ++q)
        ptx::mbar_wait(full(q % stages), (uint32_t)(q / stages) & 1u, status);
    }
    return;
  }
  // consumers: stage the NB rows of x (while the first blocks stream in)
  float* xf = reinterpret_cast<float*>(xq);
#pragma unroll 1
  for (int j = 0; j < NB; ++j) {
    const float* xr = x + ((size_t)(b0 + j) * T + (T - 1)) * ldx;
    float sq = 0.f;
    for (int c = threadIdx.x; c < C; c += 32 * kLastConsumers) {
      const float v = xr[c];
      sq += v * v;
      const int ci = c / kN, e = c % kN;
      xf[(((size_t)j * kH + e / 4) * nchunks + ci) * 4 + (e & 3)] = static_cast<float>(Chunk<TW>::round(v));
    }
    sq = warp_sum(sq);
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kLastConsumers));
    if (lane == 0) red[warp] = sq;
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kLastConsumers));
    if (threadIdx.x == 0) {
      float t = 0.f;
      for (int w = 0; w < kLastConsumers; ++w) t += red[w];
      rs[j] = rsqrtf(t / (float)C + eps);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(32 * kLastConsumers));
  const int grp = warp / kLastGroupWarps, gw = warp % kLastGroupWarps;
  const int r = kLastR * gw;  // this warp's rows within a block
  int k = grp;
  for (int blk = blockIdx.x + grp * gridDim.x; blk < nblk; blk += 2 * gridDim.x, k += 2) {
    const int s = k % stages;
    if (abort_flag || !ptx::mbar_wait(full(s), (uint32_t)(k / stages) & 1u, status)) { abort_flag = 1; break; }
    const int r0 = blk * rows;
    const int nr = V - r0 < rows ? V - r0 : rows;
    if (r < nr) {
      const int nq = nr - r < kLastR ? nr - r : kLastR;  // rows of this warp inside the block
      const uint4* wr[kLastR];
#pragma unroll
      for (int q = 0; q < kLastR; ++q)  // rows past the block's end repeat row r (their sums are dropped)
        wr[q] = reinterpret_cast<const uint4*>(ring + s * stage_bytes + (size_t)(r + (q < nq ? q : 0)) * row_bytes);
      float2 acc[kLastR][NB];
#pragma unroll
      for (int q = 0; q < kLastR; ++q)
#pragma unroll
        for (int j = 0; j < NB; ++j) acc[q][j] = make_float2(0.f, 0.f);
#pragma unroll 2
      for (int ci = lane; ci < nchunks; ci += 32) {
        float2 wf[kLastR][kN / 2];
#pragma unroll
        for (int q = 0; q < kLastR; ++q) Chunk<TW>::unpack(wr[q][ci], wf[q]);
#pragma unroll
        for (int j = 0; j < NB; ++j) {
#pragma unroll
          for (int h = 0; h < kH; ++h) {
            const float4 xv = xq[((size_t)j * kH + h) * nchunks + ci];
#pragma unroll
            for (int q = 0; q < kLastR; ++q) {
              acc[q][j] = ffma2(wf[q][2 * h], make_float2(xv.x, xv.y), acc[q][j]);
              acc[q][j] = ffma2(wf[q][2 * h + 1], make_float2(xv.z, xv.w), acc[q][j]);
            }
          }
        }
      }
      // value index q * kNV + j; lane l ends up with the total of one of them
      float vals[1 << kK];
#pragma unroll
      for (int q = 0; q < kLastR; ++q)
#pragma unroll
        for (int j = 0; j < kNV; ++j) vals[q * kNV + j] = j < NB ? acc[q][j].x + acc[q][j].y : 0.f;
      const float tot = warp_reduce_many<kK>(vals, lane);
      int vi = 0;
#pragma unroll
      for (int rr = 0; rr < kK; ++rr) vi |= ((lane >> (4 - rr)) & 1) << (kK - 1 - rr);
      const int q = vi / kNV, j = vi % kNV;
      const bool writer = (lane & ((1 << (5 - kK)) - 1)) == 0;
      if (writer && j < NB && q < nq)
        out[(size_t)(b0 + j) * ldo + r0 + r + q] = cap * tanhf(tot * rs[j] / cap);
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(empty(s));
  }
}

// ---------------------------------------------------------------------------
// Last-position logits on the tensor cores (bf16 W_U, C a multiple of 64)
// ---------------------------------------------------------------------------
// The same product as k_last_logits, logits^T = W_U x^T, as an MMA with the
// vocabulary rows as M and the (at most 16) x rows as N:
//   * x^T is staged once per CTA in shared memory as the B operand (bf16,
//     K-major, 128-byte swizzle: for each 64-wide k block, 16 rows of 128 B);
//   * W_U streams through a ring of stages by TMA, one 32-row x 64-k box per
//     32-row unit (128-byte swizzle); a stage holds the 4 to 8 units a CTA
//     takes per pass, covered by one or two M = 128 tiles (the second one
//     ends at the last unit, overlapping the first);
//   * one thread issues tcgen05.mma (M = 128, N = 16, K = 16) into TMEM; four
//     epilogue warps read D (lane = vocabulary row, column = x row), apply
//     the RMSNorm scale and the softcap, and each lane stores its vocabulary
//     row's logit for every x row, so a warp's stores for one x row are 128
//     contiguous bytes.
// Each CTA owns a contiguous run of units (the units spread evenly over the
// grid), taken in passes of 4 to 8 units (the stage size) with two TMEM
// buffers.  W_U does not depend on the previous kernel, so the copy thread
// issues the first three stages before the programmatic-dependency wait
// clears; it issues the rest once the staging threads have sent out their x
// loads, so that those do not queue behind a full ring of W_U copies (the
// first MMA needs x^T).  Every wait is bounded; on a timeout the CTA records
// NC_ERR_TIMEOUT and returns once its copies and MMAs have landed.
constexpr int kLtUnit = 32;                                 // vocabulary rows per TMA box
constexpr int kLtUnitsMax = 8;                              // units per pass (two M = 128 tiles)
constexpr int kLtN = 16;                                    // MMA N: x rows of one launch
constexpr int kLtBoxBytes = kLtUnit * 128;                  // 4 KB: 32 rows x 64 bf16
constexpr int kLtMaxStages = 8;
constexpr int kLtThreads = 192;                             // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr uint32_t kLtTmemCols = 64;                        // 2 buffers x 2 tiles x 16 columns

constexpr int kLtSmemLimit = 227 * 1024;

// su: units per pass (and per stage), from the units a CTA of the grid takes,
// at least 4 (one full M = 128 tile) and at most 8; stages: as many as fit.
struct LtGeom {
  int su, stages;
  size_t xt_bytes, stage_bytes, smem;
};
inline LtGeom lt_geom(int C, int V, int grid) {
  LtGeom g;
  const int nunits = (V + kLtUnit - 1) / kLtUnit;
  const int per_cta = grid > 0 ? (nunits + grid - 1) / grid : kLtUnitsMax;
  g.su = per_cta < 4 ? 4 : (per_cta > kLtUnitsMax ? kLtUnitsMax : per_cta);
  g.xt_bytes = (size_t)kLtN * C * 2;
  g.stage_bytes = (size_t)g.su * kLtBoxBytes;
  // (256 bytes of the limit are left to the kernel's static shared memory)
  const size_t limit = kLtSmemLimit - 256, fixed = 1024 + 256;
  const size_t avail = limit > fixed + g.xt_bytes ? limit - fixed - g.xt_bytes : 0;
  g.stages = (int)(avail / g.stage_bytes);
  if (g.stages > kLtMaxStages) g.stages = kLtMaxStages;
  g.smem = fixed + g.xt_bytes + (size_t)g.stages * g.stage_bytes;
  return g;
}

__global__ void __launch_bounds__(kLtThreads, 1)
k_last_logits_tc(const __grid_constant__ CUtensorMap tmW, const float* __restrict__ x, int ldx, int T, int b0, int nb,
                 int V, int C, float cap, float eps, float* __restrict__ out, int ldo, int su, int stages,
                 int* status) {
  pdl_launch_dependents();
  extern __shared__ uint8_t lt_raw[];
  const size_t stage_bytes = (size_t)su * kLtBoxBytes;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lt_raw) + 1023) & ~uintptr_t(1023));
  const int nkb = C / 64;
  uint8_t* xt = smem;                                   // nkb blocks of 2 KB
  uint8_t* ring = smem + (size_t)kLtN * C * 2;          // a multiple of 2 KB past a 1 KB boundary
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + (size_t)stages * stage_bytes);
  // full[kLtMaxStages] | empty[kLtMaxStages] | tfull[2] | tempty[2] | done
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kLtMaxStages + s); };
  auto tfull = [&](int b) { return bar0 + 8u * (2 * kLtMaxStages + b); };
  auto tempty = [&](int b) { return bar0 + 8u * (2 * kLtMaxStages + 2 + b); };
  const uint32_t done = bar0 + 8u * (2 * kLtMaxStages + 4);
  const uint32_t xbar = bar0 + 8u * (2 * kLtMaxStages + 5);  // the staging threads' x loads are issued
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kLtMaxStages + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ float ssq[kLtN];  // sum of squares of each x row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x < kLtN) ssq[threadIdx.x] = 0.f;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull(b), 1);
      ptx::mbar_init(tempty(b), 4);
    }
    ptx::mbar_init(done, 1);
    ptx::mbar_init(xbar, 32 * 5);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kLtTmemCols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  // this CTA's units [u_lo, u_hi) of 32 vocabulary rows
  const int nunits = (V + kLtUnit - 1) / kLtUnit;
  const int u_lo = (int)((long long)blockIdx.x * nunits / gridDim.x);
  const int u_hi = (int)((long long)(blockIdx.x + 1) * nunits / gridDim.x);
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer (reads only W_U: no dependency wait) ----------------
    if (ptx::elect_one()) {
      int k = 0;
      bool ok = true;
      const int early = min(3, stages);  // stages issued before the x loads
      for (int ub = u_lo; ub < u_hi && ok; ub += su) {
        const int nu = min(su, u_hi - ub);
        for (int kb = 0; kb < nkb; ++kb, ++k) {
          const int s = k % stages;
          if (k == early && !ptx::mbar_wait(xbar, 0, status)) {
            ok = false;
            break;
          }
          if (*abort_flag || !ptx::mbar_wait(empty(s), ((uint32_t)(k / stages) & 1u) ^ 1u, status)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(full(s), (uint32_t)(nu * kLtBoxBytes));
          const uint32_t dst = ptx::smem_u32(ring + (size_t)s * stage_bytes);
          for (int i = 0; i < nu; ++i)
            ptx::tma_load_2d(dst + (uint32_t)(i * kLtBoxBytes), &tmW, full(s), kb * 64, (ub + i) * kLtUnit);
        }
      }
      if (!ok) *abort_flag = 1;
      // every issued copy has landed before the CTA may exit
      for (int q = k - stages > 0 ? k - stages : 0; q < k; ++q)
        ptx::mbar_wait(full(q % stages), (uint32_t)(q / stages) & 1u, status);
    }
  } else {
    pdl_wait();  // x comes from the previous kernel
    // ---------------- stage x^T (warps 1..5) ----------------
    // The chunks (8 consecutive k, 16 bytes of bf16) of all rows are spread
    // over the 160 threads; each thread issues the loads of up to five
    // chunks before it uses any of them, so the staging costs about one
    // memory round trip per round rather than one per chunk.
    const int tid = threadIdx.x - 32, nth = 32 * 5;
    const int cpr = C / 8;
    auto chunk_at = [&](int j, int ci) {
      return reinterpret_cast<uint4*>(xt + (size_t)(ci >> 3) * 2048 + j * 128 + (((ci & 7) ^ (j & 7)) << 4));
    };
    for (int t = tid; t < (kLtN - nb) * cpr; t += nth) *chunk_at(nb + t / cpr, t % cpr) = make_uint4(0u, 0u, 0u, 0u);
    constexpr int U = 5;  // d24 widths, four rows: 768 chunks, one round over 160 threads
    for (int t0 = tid, round = 0; t0 < nb * cpr || round == 0; t0 += U * nth, ++round) {
      float4 va[U], vb[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * nth;
        va[u] = vb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < nb * cpr) {
          const float* xr = x + ((size_t)(b0 + t / cpr) * T + (T - 1)) * ldx + 8 * (t % cpr);
          va[u] = *reinterpret_cast<const float4*>(xr);
          vb[u] = *reinterpret_cast<const float4*>(xr + 4);
        }
      }
      if (round == 0) ptx::mbar_arrive_relaxed(xbar);  // every staging thread, once
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * nth;
        const bool live = t < nb * cpr;
        float sq = 0.f;
        if (live) {
          const float4 a = va[u], b = vb[u];
          sq = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w + b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
          const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
          const __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
          *chunk_at(t / cpr, t % cpr) =
              make_uint4(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1),
                         *reinterpret_cast<const uint32_t*>(&p2), *reinterpret_cast<const uint32_t*>(&p3));
        }
        if (cpr % 32 == 0) {
          // a warp's 32 consecutive chunks lie in one row and are all live
          // or all not: one shared-memory atomic per warp, not 32 on one word
          sq = warp_sum(sq);
          if (lane == 0 && live) atomicAdd(&ssq[t / cpr], sq);
        } else if (live) {
          atomicAdd(&ssq[t / cpr], sq);
        }
      }
    }
    ptx::fence_proxy_async_smem();  // the tensor core reads x^T through the async proxy
    asm volatile("bar.sync 1, %0;" ::"r"(32 * 5));

    if (warp == 1) {
      // ---------------- MMA issuer ----------------
      if (ptx::elect_one()) {
        constexpr uint32_t idesc = ptx::idesc_bf16(128, kLtN);
        const uint32_t xt0 = ptx::smem_u32(xt);
        int k = 0, pass = 0;
        bool ok = true;
        for (int ub = u_lo; ub < u_hi && ok; ub += su, ++pass) {
          const int nu = min(su, u_hi - ub);
          const int buf = pass & 1;
          if (*abort_flag || !ptx::mbar_wait(tempty(buf), ((uint32_t)(pass >> 1) & 1u) ^ 1u, status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(buf * 2 * kLtN);
          for (int kb = 0; kb < nkb; ++kb, ++k) {
            const int s = k % stages;
            if (*abort_flag || !ptx::mbar_wait(full(s), (uint32_t)(k / stages) & 1u, status)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint32_t a0 = ptx::smem_u32(ring + (size_t)s * stage_bytes);
            // the second tile covers the pass's last 128 rows (units nu - 4 .. nu - 1)
            const uint32_t a1 = a0 + (uint32_t)((nu - 4) * kLtBoxBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = ptx::desc_kmajor_sw128(xt0 + (uint32_t)(kb * 2048 + kk * 32));
              const uint32_t acc = (kb | kk) != 0;
              ptx::mma_bf16_ss(d, ptx::desc_kmajor_sw128(a0 + (uint32_t)(kk * 32)), bd, idesc, acc);
              if (nu > 4)
                ptx::mma_bf16_ss(d + kLtN, ptx::desc_kmajor_sw128(a1 + (uint32_t)(kk * 32)), bd, idesc, acc);
            }
            ptx::mma_commit(empty(s));
          }
          if (ok) ptx::mma_commit(tfull(buf));
        }
        if (!ok) *abort_flag = 1;
        // every issued MMA has completed before TMEM is released
        ptx::mma_commit(done);
        ptx::mbar_wait(done, 0, status);
      }
    } else {
      // ---------------- epilogue (warps 2..5) ----------------
      const int q = warp & 3;  // TMEM lane quarter this warp may access
      float rs[kLtN];          // 1 / rms of each x row
#pragma unroll
      for (int j = 0; j < kLtN; ++j) rs[j] = rsqrtf(ssq[j] / (float)C + eps);
      int pass = 0;
      for (int ub = u_lo; ub < u_hi; ub += su, ++pass) {
        const int nu = min(su, u_hi - ub);
        const int buf = pass & 1;
        if (*abort_flag || !ptx::mbar_wait(tfull(buf), (uint32_t)(pass >> 1) & 1u, status)) {
          *abort_flag = 1;
          break;
        }
        ptx::tc_fence_after();
        const int row_end = min((ub + nu) * kLtUnit, V);
        for (int t = 0; t < (nu > 4 ? 2 : 1); ++t) {
          uint32_t r[16];
          ptx::tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * 2 * kLtN + t * kLtN), r);
          ptx::tmem_ld_wait();
          // row of the pass: tile 0 holds rows 0..127, tile 1 rows (nu - 4) * 32 .. nu * 32 - 1,
          // of which it stores those past 127
          const int rp = (t == 0 ? 0 : (nu - 4) * kLtUnit) + q * 32 + lane;
          const int row = ub * kLtUnit + rp;
          if (row < row_end && (t == 0 || rp >= 128)) {
#pragma unroll
            for (int j = 0; j < kLtN; ++j)
              if (j < nb)
                out[(size_t)(b0 + j) * ldo + row] = cap * tanhf(__uint_as_float(r[j]) * rs[j] / cap);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(tempty(buf));
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kLtTmemCols);
  }
}

// ---------------------------------------------------------------------------
// sampling, one CTA of 1024 threads per row
// ---------------------------------------------------------------------------

constexpr int kSampleThreads = 1024;
// a row of up to this many bytes of logits is staged in shared memory
constexpr size_t kSampleSmemMax = 160 * 1024;

// order-preserving map of a float to an unsigned key (larger float, larger
// key); -0 maps with +0, as the two compare equal
__device__ __forceinline__ uint32_t fkey(float f) {
  uint32_t u = __float_as_uint(f);
  u = (u == 0x80000000u) ? 0u : u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unkey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// keys of the top digit's bin kept for the lower digits of the radix select
constexpr int kCand = 4096;

__global__ void __launch_bounds__(kSampleThreads, 1)
k_sample(const float* __restrict__ logits, int V, int ldl, float temperature, int top_k,
         const float* __restrict__ uniforms, int32_t* __restrict__ out, int in_smem, int* status) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) unsigned char sh_raw[];
  uint32_t* cand = reinterpret_cast<uint32_t*>(sh_raw);       // [kCand]
  float* zsh = reinterpret_cast<float*>(sh_raw + kCand * 4);  // [V] when the row is staged
  __shared__ uint32_t hist[256];
  __shared__ uint32_t whist[32][256];  // one digit histogram per warp
  __shared__ uint32_t s_key[32];
  __shared__ int s_idx[32];
  __shared__ float wtot[32];
  __shared__ uint32_t s_sel[2];
  __shared__ uint32_t s_ncand;
  __shared__ int s_pick;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const float* zg = logits + (size_t)b * ldl;
  const float* z = in_smem ? zsh : zg;
  // stage the row and find its largest entry (greedy answer; lowest index
  // among equal maxima) in one pass
  uint32_t bk = 0u;
  int bi = 0x7fffffff;
  for (int i = tid; i < V; i += kSampleThreads) {
    const float zi = zg[i];
    if (in_smem) zsh[i] = zi;
    const uint32_t k = fkey(zi);
    if (k > bk || (k == bk && i < bi)) { bk = k; bi = i; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t k2 = __shfl_xor_sync(0xffffffffu, bk, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
    if (k2 > bk || (k2 == bk && i2 < bi)) { bk = k2; bi = i2; }
  }
  if (lane == 0) { s_key[wid] = bk; s_idx[wid] = bi; }
  __syncthreads();
  if (wid == 0) {
    bk = s_key[lane];
    bi = s_idx[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t k2 = __shfl_xor_sync(0xffffffffu, bk, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
      if (k2 > bk || (k2 == bk && i2 < bi)) { bk = k2; bi = i2; }
    }
    if (lane == 0) { s_key[0] = bk; s_idx[0] = bi; }
  }
  __syncthreads();
  const uint32_t kmax = s_key[0];
  const int imax = s_idx[0];
  if (!(temperature > 0.f)) {
    if (tid == 0) out[b] = imax;
    return;
  }
  // top-k threshold: the key of the k-th largest entry (ties counted), found
  // digit by digit from the most significant byte
  uint32_t thr = 0u;
  if (top_k > 0 && top_k < V) {
    // histogram of digit (key >> shift) & 255 over the keys with
    // (key & pmask) == prefix, taken from the row or from the candidate list
    auto count = [&](int shift, uint32_t prefix, uint32_t pmask, bool from_cand, int n) {
      for (int i = tid; i < 32 * 256; i += kSampleThreads) (&whist[0][0])[i] = 0u;
      __syncthreads();
      for (int i0 = 0; i0 < n; i0 += kSampleThreads) {
        const int i = i0 + tid;
        uint32_t k = 0u;
        bool in = false;
        if (i < n) {
          k = from_cand ? cand[i] : fkey(z[i]);
          in = (k & pmask) == prefix;
        }
        if (__any_sync(0xffffffffu, in)) {
          const uint32_t d = in ? (k >> shift) & 255u : 0xffffffffu;  // lanes out form one group
          // lanes with the same digit add once, through their leader, into
          // this warp's own histogram (no contention between warps)
          const uint32_t peers = __match_any_sync(0xffffffffu, d);
          if (in && (__ffs(peers) - 1) == lane) whist[wid][d] += (uint32_t)__popc(peers);
        }
      }
      __syncthreads();
      if (tid < 256) {
        uint32_t t = 0u;
#pragma unroll 8
        for (int w = 0; w < 32; ++w) t += whist[w][tid];
        hist[tid] = t;
      }
      __syncthreads();
    };
    // the digit whose bin holds the rank-th largest key, and the rank within it
    auto select = [&](uint32_t rank) {
      if (wid == 0) {
        // lane l owns digits 255 - 8 l down to 248 - 8 l
        uint32_t cnt[8], tot = 0u;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cnt[e] = hist[255 - 8 * lane - e];
          tot += cnt[e];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const uint32_t excl = incl - tot;
        if (excl < rank && rank <= incl) {
          uint32_t c = excl;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (c + cnt[e] >= rank) {
              s_sel[0] = (uint32_t)(255 - 8 * lane - e);
              s_sel[1] = rank - c;
              break;
            }
            c += cnt[e];
          }
        }
      }
      __syncthreads();
    };
    count(24, 0u, 0u, false, V);
    select((uint32_t)top_k);
    uint32_t prefix = s_sel[0] << 24, pmask = 0xff000000u, rank = s_sel[1];
    const uint32_t nbin = hist[s_sel[0]];
    const bool use_cand = nbin <= (uint32_t)kCand;
    __syncthreads();
    if (use_cand) {
      // compact the keys of the selected bin (warp-aggregated slots)
      if (tid == 0) s_ncand = 0u;
      __syncthreads();
      for (int i0 = 0; i0 < V; i0 += kSampleThreads) {
        const int i = i0 + tid;
        const uint32_t k = i < V ? fkey(z[i]) : 0u;
        const bool in = i < V && (k & pmask) == prefix;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        if (m) {
          const int leader = __ffs(m) - 1;
          uint32_t base = 0u;
          if (lane == leader) base = atomicAdd(&s_ncand, (uint32_t)__popc(m));
          base = __shfl_sync(0xffffffffu, base, leader);
          if (in) cand[base + __popc(m & ((1u << lane) - 1u))] = k;
        }
      }
      __syncthreads();
    }
    const int n = use_cand ? (int)nbin : V;
    for (int shift = 16; shift >= 0; shift -= 8) {
      count(shift, prefix, pmask, use_cand, n);
      select(rank);
      prefix |= s_sel[0] << shift;
      pmask |= 255u << shift;
      rank = s_sel[1];
      __syncthreads();
    }
    thr = prefix;
  }
  // weights w_i = exp((z_i - z_max) / tau) over the kept entries.  Warp w owns
  // the contiguous indices [w bw, (w + 1) bw) and walks them 32 at a time
  // (lane l reads index i0 + l: conflict-free); steps with no kept entry cost
  // one ballot.
  const float zmax = unkey(kmax);
  const float itau = 1.0f / temperature;
  const int nw = kSampleThreads / 32;
  const int bw = ((V + nw - 1) / nw + 31) & ~31;
  const int wlo = min(wid * bw, V), whi = min(wlo + bw, V);
  float acc = 0.f;
  int lastpos = -1;  // last index of this warp's block with a positive weight
  for (int i0 = wlo; i0 < whi; i0 += 32) {
    const int i = i0 + lane;
    const float zi = i < whi ? z[i] : 0.f;
    const bool kept = i < whi && fkey(zi) >= thr;
    if (__ballot_sync(0xffffffffu, kept)) {
      const float wi = kept ? expf((zi - zmax) * itau) : 0.f;
      acc += wi;
      const uint32_t pos = __ballot_sync(0xffffffffu, wi > 0.f);
      if (pos) lastpos = i0 + 31 - __clz(pos);
    }
  }
  const float run = warp_sum(acc);
  if (lane == 0) { wtot[wid] = run; s_idx[wid] = lastpos; }
  __syncthreads();
  float u = uniforms[b];
  if (!(u >= 0.f && u < 1.f)) {
    if (tid == 0) atomicOr(status, kStatusData);
    u = fminf(fmaxf(u, 0.f), 0.99999994f);
  }
  if (tid == 0) {
    // warp prefixes in warp order; the draw falls in the first warp (with a
    // positive sum) whose inclusive prefix exceeds u * total
    float total = 0.f;
    for (int w = 0; w < nw; ++w) total += wtot[w];
    const float target = u * total;
    float c = 0.f;
    int pick_w = -1, last_w = -1;
    for (int w = 0; w < nw; ++w) {
      if (wtot[w] > 0.f) {
        last_w = w;
        if (pick_w < 0 && c + wtot[w] > target) {
          pick_w = w;
          s_sel[1] = __float_as_uint(c);  // prefix before the drawing warp
        }
      }
      c += wtot[w];
    }
    s_sel[0] = __float_as_uint(target);
    // none passes (u * total at the very top, by rounding): the last token
    // with a positive weight
    s_pick = pick_w >= 0 ? -1 - pick_w : (last_w >= 0 ? s_idx[last_w] : imax);
  }
  __syncthreads();
  if (s_pick < 0 && wid == -1 - s_pick) {
    // walk the drawing warp's block again, step by step, and pick the first
    // lane whose running prefix passes the target; if rounding leaves none,
    // the block's last token with a positive weight
    const float target = __uint_as_float(s_sel[0]);
    float c = __uint_as_float(s_sel[1]);
    int pick = lastpos;
    for (int i0 = wlo; i0 < whi; i0 += 32) {
      const int i = i0 + lane;
      const float zi = i < whi ? z[i] : 0.f;
      const bool kept = i < whi && fkey(zi) >= thr;
      if (!__ballot_sync(0xffffffffu, kept)) continue;
      const float wi = kept ? expf((zi - zmax) * itau) : 0.f;
      float inc = wi;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float nb = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += nb;
      }
      const uint32_t past = __ballot_sync(0xffffffffu, wi > 0.f && c + inc > target);
      if (past) {
        pick = i0 + __ffs(past) - 1;
        break;
      }
      c += warp_sum(wi);
    }
    if (lane == 0) out[b] = pick;
  } else if (s_pick >= 0 && tid == 0) {
    out[b] = s_pick;
  }
}

template <typename TW, int NB>
void launch_last_logits_nb(const float* x, int ldx, int T, int b0, const TW* W, int V, int C, float cap, float eps,
                           float* out, int ldo, int num_sms, int* status, cudaStream_t st) {
  const LastGeom g = last_geom(C, (int)sizeof(TW), NB);
  // a failure here leaves the launch to fail, which the entry point reports
  if (!smem_optin(k_last_logits<TW, NB>, 220 * 1024)) return;
  launch_pdl(k_last_logits<TW, NB>, dim3(num_sms), dim3(kLastThreads), g.smem, st, 1, x, ldx, T, b0, W, V, C, cap,
             eps, out, ldo, g.stages, status);
}

template <typename TW>
void launch_last_logits_t(const float* x, int ldx, int B, int T, const TW* W, int V, int C, float cap, float eps,
                          float* out, int ldo, int num_sms, int* status, cudaStream_t st) {
  for (int b0 = 0; b0 < B; b0 += kLastRows) {
    const int nb = B - b0 < kLastRows ? B - b0 : kLastRows;
    LaunchScope scope_(KK_LAST_LOGITS, st);
    switch (nb) {
      case 1: launch_last_logits_nb<TW, 1>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
      case 2: launch_last_logits_nb<TW, 2>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
      case 3: launch_last_logits_nb<TW, 3>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
      case 4: launch_last_logits_nb<TW, 4>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
      case 5: launch_last_logits_nb<TW, 5>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
      case 6: launch_last_logits_nb<TW, 6>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
      case 7: launch_last_logits_nb<TW, 7>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
      default: launch_last_logits_nb<TW, 8>(x, ldx, T, b0, W, V, C, cap, eps, out, ldo, num_sms, status, st); break;
    }
  }
}

}  // namespace

// The tensor-core form: bf16 W_U with C a multiple of 64 and room for two
// ring stages next to x^T.  False when it does not apply or its tensor map
// cannot be made (the CUDA-core form then runs).
static bool launch_last_logits_tc(const float* x, int ldx, int B, int T, const bf16* W, int V, int C, float cap, float eps,
                           float* out, int ldo, int num_sms, int* status, cudaStream_t st) {
  if (C % 64 != 0 || V <= 0 || ldx % 4 != 0) return false;
  const LtGeom g = lt_geom(C, V, num_sms);
  if (g.stages < 2) return false;
  CUtensorMap tm;
  if (!make_tmap_2d(&tm, W, V, C, C, kLtUnit, 64)) return false;
  if (!smem_optin(k_last_logits_tc, (int)g.smem)) return false;
  for (int b0 = 0; b0 < B; b0 += kLtN) {
    const int nb = B - b0 < kLtN ? B - b0 : kLtN;
    LaunchScope scope_(KK_LAST_LOGITS, st);
    launch_pdl(k_last_logits_tc, dim3(num_sms), dim3(kLtThreads), g.smem, st, 1, tm, x, ldx, T, b0, nb, V, C, cap, eps,
               out, ldo, g.su, g.stages, status);
  }
  return true;
}

void launch_last_logits(const float* x, int ldx, int B, int T, const void* W, int V, int C, bool bf, float cap,
                        float eps, float* out, int ldo, int num_sms, int* status, cudaStream_t st) {
  if (bf && launch_last_logits_tc(x, ldx, B, T, static_cast<const bf16*>(W), V, C, cap, eps, out, ldo, num_sms,
                                  status, st))
    return;
  if (bf)
    launch_last_logits_t(x, ldx, B, T, static_cast<const bf16*>(W), V, C, cap, eps, out, ldo, num_sms, status, st);
  else
    launch_last_logits_t(x, ldx, B, T, static_cast<const float*>(W), V, C, cap, eps, out, ldo, num_sms, status, st);
}

bool last_logits_supported(int C, bool bf) {
  // bf16 with C a multiple of 64: the tensor-core form, whose stages hold at
  // most 8 units (its geometry for a grid that gives each CTA 8 units or more)
  if (bf && C > 0 && C % 64 == 0 && lt_geom(C, kLtUnitsMax * kLtUnit, 1).stages >= 2) return true;
  // otherwise the CUDA-core form: two ring stages next to eight staged rows of x
  return C > 0 && last_geom(C, bf ? 2 : 4, kLastRows).stages >= 2;
}

static bool sample_in_smem(int V) { return (size_t)V * 4 <= kSampleSmemMax; }

void launch_sample(const float* logits, int B, int V, int ldl, float temperature, int top_k,
                   const float* uniforms, int32_t* out, int* status, cudaStream_t st) {
  LaunchScope scope_(KK_SAMPLE, st);
  if (!smem_optin(k_sample, (int)(kSampleSmemMax + kCand * 4))) return;
  const bool sm = sample_in_smem(V);
  launch_pdl(k_sample, dim3(B), dim3(kSampleThreads), (size_t)kCand * 4 + (sm ? (size_t)V * 4 : 0), st, 1, logits, V,
             ldl, temperature,
             top_k, uniforms, out, sm ? 1 : 0, status);
}

}  // namespace nc
