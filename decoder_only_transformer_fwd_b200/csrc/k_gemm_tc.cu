// tcgen05 GEMM for sm_100a: C[M, N] = A[M, K] B[N, K]^T with bf16 operands
// and fp32 accumulation in tensor memory, followed by a fused epilogue.
//
// Structure (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: A and B k-slices (64 wide, 128-byte swizzle)
//               into a STAGES-deep shared-memory ring;
//   warp 1      allocates 2*BN TMEM columns; one thread issues tcgen05.mma
//               (M = 128, N = BN, K = 16) into one of two accumulators;
//   warps 2..9  epilogue, two warps per TMEM lane quarter (one TMEM lane per
//               output row), each on half of the tile's columns: tcgen05.ld of
//               the accumulator, the fused element-wise op, global stores.
// The kernel is specialised on the epilogue at compile time.
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

#include <string.h>

#include <mutex>

#include "epilogue.cuh"
#include "ptx.cuh"

namespace nc {

namespace {

constexpr int kBM = 128, kBK = 64, kUK = 16;
constexpr int kEpiWarps = 8;                 // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;  // + the TMA and MMA warps

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
  static constexpr int EPI_BYTES = kEpiWarps * STAGE_FLOATS * 4;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256 + EPI_BYTES;
};

struct TcArgs {
  int M, N, K;
  int tiles_m, tiles_n, num_tiles;
  int n_fastest;  // pair kernel: tile order with the column tile varying fastest
  int* status;
  // pair kernel, stream-K schedule (see PairSched); sk_ws holds one fp32
  // partial accumulator per CTA (128 x 256, column-major), sk_flags one word
  // per CTA, set to sk_gen once that CTA's partial is written; a finishing
  // pair waits (at most sk_wait_ns) until its contributors' flags equal
  // sk_expect, which is sk_gen except under the timeout test hook
  int streamk;
  float* sk_ws;
  unsigned* sk_flags;
  unsigned sk_gen;
  unsigned sk_expect;
  unsigned long long sk_wait_ns;
  // pair kernel, block lower triangular B (kl_k > 0): output columns below
  // kl_out_end[a] read only the first kl_in_end[a] elements of K, so a column
  // tile's contraction stops after the K prefix its last column reads
  int kl_k;
  int kl_out_end[kMaxPrefixBlocks];
  int kl_in_end[kMaxPrefixBlocks];
};

// The k-blocks a pair column tile nb (width bn) contracts over: all of K, or
// with a block lower triangular B the prefix its last column reads.
__device__ __forceinline__ int tile_kb_end(const TcArgs& a, int nb, int bn, int nk) {
  if (a.kl_k <= 0) return nk;
  const int lc = min(a.N, (nb + 1) * bn) - 1;
  int kend = a.K;
#pragma unroll
  for (int i = kMaxPrefixBlocks - 1; i >= 0; --i)
    if (i < a.kl_k && a.kl_out_end[i] > lc) kend = a.kl_in_end[i];
  const int kb = (kend + kBK - 1) / kBK;
  return kb < nk ? kb : nk;
}

// Pair tile pt -> (row-pair block, column tile).  Column-fastest order keeps
// the A rows that the CTAs of one wave share few enough to stay in L2 (for
// GEMMs whose B is the smaller operand); row-fastest order does the same for
// B (the head, whose weight is the larger operand).
__device__ __forceinline__ void pair_tile(const TcArgs& a, int pt, int tiles_mp, int& mbp, int& nb) {
  if (a.n_fastest) {
    mbp = pt / a.tiles_n;
    nb = pt % a.tiles_n;
  } else {
    mbp = pt % tiles_mp;
    nb = pt / tiles_mp;
  }
}

// Work of one CTA pair (cluster cid of ncl): njobs jobs, job j being pair
// tile pt with k-blocks [kb_lo, kb_hi).  Plain schedule: tiles cid, cid + ncl,
// ... with all k-blocks.  Stream-K schedule (data-parallel waves plus a split
// tail): the W = num_pt / ncl full waves stay as they are (so the tiles in
// flight at any time share their A rows in L2), and the k-blocks of the
// num_pt % ncl tiles of the last, partial wave are cut into ncl equal ranges,
// one per pair.  A range lies within one tile or spans the end of one tile
// and the start of the next.  The pair whose range holds a tile's last
// k-block finishes that tile (its "owner" job) after adding the partial sums
// of the pairs before it that hold the tile's earlier k-blocks
// ("contributor" jobs).  Order per pair: contributor job first, full waves,
// owner job last, so the partials are written long before they are needed.
struct PairSched {
  int streamk, nk, cid, ncl, waves, tail_pt0;
  long long u0, u1;        // this pair's range of tail (tile, k-block) units
  int contrib, owner;      // has a contributor job / an owner job
  int njobs;
};

__device__ __forceinline__ PairSched make_sched(const TcArgs& a, int num_pt, int nk, int cid, int ncl) {
  PairSched s;
  s.streamk = a.streamk;
  s.nk = nk;
  s.cid = cid;
  s.ncl = ncl;
  s.waves = num_pt / ncl;
  s.tail_pt0 = s.waves * ncl;
  s.u0 = s.u1 = 0;
  s.contrib = s.owner = 0;
  if (!a.streamk) {
    s.njobs = cid < num_pt ? (num_pt - cid + ncl - 1) / ncl : 0;
    return s;
  }
  const long long U = (long long)(num_pt - s.tail_pt0) * nk;
  s.u0 = U * cid / ncl;
  s.u1 = U * (cid + 1) / ncl;
  if (s.u1 > s.u0) {
    s.contrib = (s.u1 % nk) != 0;                                   // range ends inside a tile
    s.owner = (s.u1 - s.u0) > (s.contrib ? s.u1 % nk : 0);          // it also holds some tile's end
  }
  s.njobs = s.contrib + s.waves + s.owner;
  return s;
}

// kind: 0 full tile, 1 contributor (writes a partial), 2 owner (adds partials)
__device__ __forceinline__ void job_at(const PairSched& s, int j, int& pt, int& kb_lo, int& kb_hi, int& kind) {
  kind = 0;
  if (!s.streamk) {
    pt = s.cid + j * s.ncl;
    kb_lo = 0;
    kb_hi = s.nk;
    return;
  }
  if (s.contrib && j == 0) {  // the start of the tile holding this range's end
    const long long tt = (s.u1 - 1) / s.nk;
    pt = s.tail_pt0 + (int)tt;
    kb_lo = (int)(s.u0 > tt * s.nk ? s.u0 - tt * s.nk : 0);
    kb_hi = (int)(s.u1 - tt * s.nk);
    kind = 1;
    return;
  }
  const int w = j - s.contrib;
  if (w < s.waves) {
    pt = s.cid + w * s.ncl;
    kb_lo = 0;
    kb_hi = s.nk;
    return;
  }
  // the end of the tile holding this range's start
  const long long tt = s.u0 / s.nk;
  pt = s.tail_pt0 + (int)tt;
  kb_lo = (int)(s.u0 - tt * s.nk);
  kb_hi = s.nk;
  kind = 2;
}

// Pairs whose contributor job is in tail tile tt, i.e. whose range ends
// inside tt: a contiguous run of pairs just before the owner.
__device__ __forceinline__ int first_contributor(const PairSched& s, long long U, long long tt) {
  int c = s.cid;
  while (c > 0) {
    const long long u1p = U * c / s.ncl;  // end of pair c - 1's range
    if (u1p <= tt * s.nk) break;
    --c;
  }
  return c;
}

__device__ __forceinline__ float bits2f(uint32_t u) { return __uint_as_float(u); }

// Per-row values of a tile that do not depend on its accumulator.  They are
// loaded before the epilogue waits for the accumulator, so their memory
// latency overlaps the tile's MMAs; the rows the epilogue will read later are
// pulled into L2 at the same time.
struct RowPre {
  float rscale;  // 1 / rms of the A row (fused RMSNorm); 1 when unused
  float gate;    // QKV value heads: the value-embedding gate
  int y;         // CE / DZ: the row's target id, or -1
  int tok;       // QKV value heads: the row's token id, clamped
  float lse;     // DZ: the row's log-sum-exp
};

// The 32 x 32 chunk epilogues below receive the accumulator one row per lane
// (TMEM lane = row) and stage it in the warp's shared-memory buffer (row
// pitch 33: conflict-free both ways).  They then work on it transposed: lane
// (q = lane / 8, c4 = lane % 8) takes columns 4 c4 .. 4 c4 + 3 of rows 4 i + q,
// i = 0..7, so every global access is a 16-byte (or 8-byte) vector and the 8
// lanes of a quarter-warp cover one contiguous row segment.

// Residual epilogues (EPI_RESID, EPI_BLOCK_END): x += acc, then for
// EPI_BLOCK_END the next block's lambda x + mu x0 or the backout capture /
// subtraction.  All of the chunk's loads are issued before its first store.
// With ep.xb_out set the new x is also stored as bf16 (the next GEMM's A
// operand) and ssr[i] accumulates the sum of squares of row 4 i + q over the
// chunk's columns (the same value in the 8 lanes of the quarter-warp).
__device__ __forceinline__ void epi_resid_chunk(const EpiParams& ep, const TcArgs& a, float* stage, int row0,
                                                int n, const uint32_t (&r)[32], int lane, float (&ssr)[8]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) stage[lane * 33 + i] = __uint_as_float(r[i]);
  __syncwarp();
  const int q = lane >> 3, c4 = lane & 7;
  const int col = n + 4 * c4;
  const bool col_ok = col + 3 < a.N;  // N is a multiple of 32 on this path
  const bool bend = ep.mode == EPI_BLOCK_END;
  const bool need_x0 = bend && ep.end_kind == 1;
  const bool need_bo = bend && ep.end_kind == 2 && !ep.capture_bo;
  const float* zsrc = need_x0 ? ep.x0 : ep.xbo;
  float lam = 1.f, mu = 0.f;
  if (need_x0) {
    lam = *ep.lam;
    mu = *ep.mu;
  }
  float4 xv[8], zv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = row0 + 4 * i + q;
    const bool ok = col_ok && m < a.M;
    const size_t off = (size_t)m * ep.ldx + col;
    xv[i] = ok ? *reinterpret_cast<const float4*>(ep.x + off) : make_float4(0.f, 0.f, 0.f, 0.f);
    zv[i] = (ok && (need_x0 || need_bo)) ? *reinterpret_cast<const float4*>(zsrc + off)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = 4 * i + q;
    const int m = row0 + rr;
    const bool ok = col_ok && m < a.M;
    const float* sr = stage + rr * 33 + 4 * c4;
    float v[4] = {xv[i].x + sr[0], xv[i].y + sr[1], xv[i].z + sr[2], xv[i].w + sr[3]};
    const float z[4] = {zv[i].x, zv[i].y, zv[i].z, zv[i].w};
    const size_t off = (size_t)m * ep.ldx + col;
    if (bend) {
      if (ep.capture_bo && ok) *reinterpret_cast<float4*>(ep.xbo + off) = make_float4(v[0], v[1], v[2], v[3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (ep.end_kind == 1)
          v[e] = lam * v[e] + mu * z[e];
        else if (ep.end_kind == 2)
          v[e] = v[e] - ep.beta * (ep.capture_bo ? v[e] : z[e]);
      }
    }
    if (ok) {
      *reinterpret_cast<float4*>(ep.x + off) = make_float4(v[0], v[1], v[2], v[3]);
      if (ep.xb_out != nullptr) {
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]), b1 = __floats2bfloat162_rn(v[2], v[3]);
        *reinterpret_cast<uint2*>(ep.xb_out + (size_t)m * ep.ldxb + col) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
      }
    }
    float sq = ok ? fmaf(v[0], v[0], fmaf(v[1], v[1], fmaf(v[2], v[2], v[3] * v[3]))) : 0.f;
    sq += __shfl_xor_sync(0xffffffffu, sq, 1);
    sq += __shfl_xor_sync(0xffffffffu, sq, 2);
    sq += __shfl_xor_sync(0xffffffffu, sq, 4);
    ssr[i] += sq;
  }
  __syncwarp();
}

// EPI_RESID, software-pipelined by the caller: resid_load requests x for a
// chunk (transposed lane layout) and resid_apply finishes a staged chunk
// with those values, so the loads of chunk c + 1 overlap the stores of c.
__device__ __forceinline__ void resid_load(const EpiParams& ep, const TcArgs& a, int row0, int n, int lane,
                                           float4 (&xv)[8]) {
  const int q = lane >> 3, c4 = lane & 7;
  const int col = n + 4 * c4;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = row0 + 4 * i + q;
    xv[i] = (col + 3 < a.N && m < a.M) ? *reinterpret_cast<const float4*>(ep.x + (size_t)m * ep.ldx + col)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}
__device__ __forceinline__ void resid_apply(const EpiParams& ep, const TcArgs& a, const float* stage, int row0,
                                            int n, int lane, const float4 (&xv)[8], float (&ssr)[8]) {
  const int q = lane >> 3, c4 = lane & 7;
  const int col = n + 4 * c4;
  const bool col_ok = col + 3 < a.N;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = 4 * i + q;
    const int m = row0 + rr;
    const bool ok = col_ok && m < a.M;
    const float* sr = stage + rr * 33 + 4 * c4;
    const float v0 = xv[i].x + sr[0], v1 = xv[i].y + sr[1], v2 = xv[i].z + sr[2], v3 = xv[i].w + sr[3];
    if (ok) {
      *reinterpret_cast<float4*>(ep.x + (size_t)m * ep.ldx + col) = make_float4(v0, v1, v2, v3);
      if (ep.xb_out != nullptr) {
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(v0, v1), b1 = __floats2bfloat162_rn(v2, v3);
        *reinterpret_cast<uint2*>(ep.xb_out + (size_t)m * ep.ldxb + col) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
      }
    }
    float sq = ok ? fmaf(v0, v0, fmaf(v1, v1, fmaf(v2, v2, v3 * v3))) : 0.f;
    sq += __shfl_xor_sync(0xffffffffu, sq, 1);
    sq += __shfl_xor_sync(0xffffffffu, sq, 2);
    sq += __shfl_xor_sync(0xffffffffu, sq, 4);
    ssr[i] += sq;
  }
}

// EPI_STORE / EPI_RELU2: rscale (this lane's row scale) and ReLU^2 are applied
// while staging; the transposed pass stores 8-byte bf16 quads.
__device__ __forceinline__ void epi_store_chunk(const EpiParams& ep, const TcArgs& a, float* stage, int row0,
                                                int n, const uint32_t (&r)[32], int lane, bool relu2,
                                                float rscale) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float v = __uint_as_float(r[i]) * rscale;
    if (relu2) {
      v = fmaxf(v, 0.f);
      v *= v;
    }
    stage[lane * 33 + i] = v;
  }
  __syncwarp();
  const int q = lane >> 3, c4 = lane & 7;
  const int col = n + 4 * c4;
  bf16* base = reinterpret_cast<bf16*>(ep.out);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = 4 * i + q;
    const int m = row0 + rr;
    const float* sr = stage + rr * 33 + 4 * c4;
    if (m < a.M) {
      bf16* dst = base + (size_t)m * ep.ldo + col;
      if (col + 3 < a.N) {
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(sr[0], sr[1]), b1 = __floats2bfloat162_rn(sr[2], sr[3]);
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (col + e < a.N) dst[e] = __float2bfloat16_rn(sr[e]);
      }
    }
  }
  __syncwarp();
}

// EPI_DZ / EPI_F32: each lane first turns its row's 32 accumulator values
// into the output value (for EPI_DZ the gradient of the mean softcapped
// cross-entropy with respect to z, scaled by the row's 1 / rms), stages them,
// and the transposed pass stores 8-byte bf16 or 16-byte fp32 quads.
template <int MODE>
__device__ __forceinline__ void epi_bwd_chunk(const EpiParams& ep, const TcArgs& a, float* stage, int row0, int n,
                                              const uint32_t (&r)[32], int lane, const RowPre& pre, float ginv) {
  if constexpr (MODE == EPI_DZ) {
    // zhat = c tanh(z / c) = c - 2c / (e^{2z/c} + 1); p = e^{zhat - lse};
    // d loss_mean / d z = (p - [n == y]) (1 - (zhat / c)^2) / count
    const float k1 = 2.0f * 1.4426950408889634f / ep.cap;
    const float c2 = -2.0f * ep.cap, inv_cap = 1.0f / ep.cap;
    const float lse2 = pre.lse * 1.4426950408889634f;
    const float scale = pre.y >= 0 ? pre.rscale * ginv : 0.f;  // ignored rows get no gradient
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float q = ptx::rcp(ptx::ex2(__uint_as_float(r[i]) * (pre.rscale * k1)) + 1.0f);
      const float zh = fmaf(c2, q, ep.cap);
      const float p = ptx::ex2(fmaf(zh, 1.4426950408889634f, -lse2));
      const float th = zh * inv_cap;
      const float d = (p - ((n + i == pre.y) ? 1.0f : 0.0f)) * (1.0f - th * th);
      stage[lane * 33 + i] = (n + i < ep.vocab) ? d * scale : 0.f;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) stage[lane * 33 + i] = __uint_as_float(r[i]);
  }
  __syncwarp();
  const int q = lane >> 3, c4 = lane & 7;
  const int col = n + 4 * c4;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = 4 * i + q;
    const int m = row0 + rr;
    const float* sr = stage + rr * 33 + 4 * c4;
    if (m < a.M) {
      if constexpr (MODE == EPI_DZ) {
        bf16* dst = reinterpret_cast<bf16*>(ep.out) + (size_t)m * ep.ldo + col;
        if (col + 3 < a.N) {
          const __nv_bfloat162 b0 = __floats2bfloat162_rn(sr[0], sr[1]), b1 = __floats2bfloat162_rn(sr[2], sr[3]);
          *reinterpret_cast<uint2*>(dst) =
              make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (col + e < a.N) dst[e] = __float2bfloat16_rn(sr[e]);
        }
      } else {
        float* dst = reinterpret_cast<float*>(ep.out) + (size_t)m * ep.ldo + col;
        if (col + 3 < a.N) {
          *reinterpret_cast<float4*>(dst) = make_float4(sr[0], sr[1], sr[2], sr[3]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (col + e < a.N) dst[e] = sr[e];
        }
      }
    }
  }
  __syncwarp();
}

// Fused QKV epilogue for the 128 columns of one head held in TMEM at taddr,
// rows m0 .. m0 + 31 (one per lane): q and k heads get RoPE (position m % T)
// and alpha * RMSNorm over the head; v heads get gate * VE[tok] added; one
// bf16 rounding at the store.  ("The Mathematics of Karpathy's nanochat",
// §Rotary Position Embeddings, §QK-Norm with Sharpening, §Value Embeddings.)
// The accumulator arrives one row per lane; it goes through the warp's
// shared-memory transpose buffer so that the RoPE table reads, the
// value-embedding reads and the output stores are row segments shared by
// groups of lanes instead of one row per lane.  Per-row values (the norm
// scale, position, token and gate) move between lanes by shuffles.
__device__ __forceinline__ void epi_qkv_head(const EpiParams& ep, const TcArgs& a, float* stage, uint32_t taddr,
                                             int m0, int lane, int col0, float rscale, float gate, int tok) {
  bf16* out = reinterpret_cast<bf16*>(ep.out) + col0;
  if (col0 < ep.qk_cols) {
    const int t_lane = (m0 + lane) % ep.T;
    const int fp = lane & 7, rsub = lane >> 3;  // lane -> (frequency pair, row within a group of 4)
    // the warp's 32 rows are 32 consecutive positions of one sequence
    const bool lin = (m0 % ep.T) + 31 < ep.T;
    const int t_first = (m0 % ep.T) + rsub;
    // RoPE pairs (j, j + 64) preserve each pair's sum of squares, so the RMS
    // comes from the raw accumulator in a first pass
    float ssa = 0.f, ssb = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t u[32];
      ptx::tmem_ld32(taddr + (uint32_t)(c * 32), u);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        ssa = fmaf(__uint_as_float(u[i]), __uint_as_float(u[i]), ssa);
        ssb = fmaf(__uint_as_float(u[i + 1]), __uint_as_float(u[i + 1]), ssb);
      }
    }
    // the head is rscale * acc: fold the row scale into the QK-norm factor
    const float rs_lane = rscale * ep.qk_alpha / sqrtf((ssa + ssb) * rscale * rscale * (1.0f / 128.0f) + ep.eps);
    // second pass over four groups of 16 frequencies; group k + 1's TMEM
    // columns are requested before group k is rotated and stored
    uint32_t r1[16], r2[16];
    ptx::tmem_ld16(taddr, r1);
    ptx::tmem_ld16(taddr + 64u, r2);
#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
      // frequencies 16k .. 16k + 15: columns 16k.. of the first half and 64 + 16k.. of the second
      ptx::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        stage[lane * 33 + i] = __uint_as_float(r1[i]);
        stage[lane * 33 + 16 + i] = __uint_as_float(r2[i]);
      }
      __syncwarp();
      if (k < 3) {
        ptx::tmem_ld16(taddr + (uint32_t)(16 * (k + 1)), r1);
        ptx::tmem_ld16(taddr + (uint32_t)(64 + 16 * (k + 1)), r2);
      }
      const int f0 = 16 * k + 2 * fp;
      // this lane's two frequencies in cycles per position, split so that the
      // phase t f mod 1 is exact to ~1e-7 (the angle then goes to the
      // hardware sine / cosine within [-pi, pi])
      const float fh0 = __ldg(ep.rope_fsplit + f0), fh1 = __ldg(ep.rope_fsplit + f0 + 1);
      const float fl0 = __ldg(ep.rope_fsplit + 64 + f0), fl1 = __ldg(ep.rope_fsplit + 64 + f0 + 1);
      // angle 2 pi (t f mod 1) of position t, |angle| <= pi
      auto angle = [&](float tf, float fh, float fl) {
        float ph = tf * fh;  // exact
        ph = fmaf(tf, fl, ph - floorf(ph));
        return (ph - rintf(ph)) * 6.2831853071795865f;
      };
      auto rotate_store = [&](int rr, float rs, float c0, float s0, float c1, float s1) {
        const float a1x = stage[rr * 33 + 2 * fp], a1y = stage[rr * 33 + 2 * fp + 1];
        const float a2x = stage[rr * 33 + 16 + 2 * fp], a2y = stage[rr * 33 + 16 + 2 * fp + 1];
        if (m0 + rr < a.M) {
          bf16* o = out + (size_t)(m0 + rr) * ep.ldo + f0;
          *reinterpret_cast<__nv_bfloat162*>(o) = __floats2bfloat162_rn((a1x * c0 + a2x * s0) * rs,
                                                                        (a1y * c1 + a2y * s1) * rs);
          *reinterpret_cast<__nv_bfloat162*>(o + 64) = __floats2bfloat162_rn((-a1x * s0 + a2x * c0) * rs,
                                                                             (-a1y * s1 + a2y * c1) * rs);
        }
      };
      if (lin) {
        // this lane's rows 4 i + rsub sit at positions t_first + 4 i: one
        // angle from the hardware sine / cosine, then exact-angle steps of
        // 4 f by rotation (7 steps add ~1e-6 to the ~4e-7 of the first angle)
        const float tf = (float)t_first;
        const float q0 = angle(tf, fh0, fl0), q1 = angle(tf, fh1, fl1);
        const float d0 = angle(4.0f, fh0, fl0), d1 = angle(4.0f, fh1, fl1);
        float c0 = __cosf(q0), s0 = __sinf(q0), c1 = __cosf(q1), s1 = __sinf(q1);
        const float dc0 = __cosf(d0), ds0 = __sinf(d0), dc1 = __cosf(d1), ds1 = __sinf(d1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + rsub;
          rotate_store(rr, __shfl_sync(0xffffffffu, rs_lane, rr), c0, s0, c1, s1);
          const float c0n = fmaf(c0, dc0, -s0 * ds0), s0n = fmaf(s0, dc0, c0 * ds0);
          const float c1n = fmaf(c1, dc1, -s1 * ds1), s1n = fmaf(s1, dc1, c1 * ds1);
          c0 = c0n;
          s0 = s0n;
          c1 = c1n;
          s1 = s1n;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + rsub;
          const float rs = __shfl_sync(0xffffffffu, rs_lane, rr);
          const float tf = (float)__shfl_sync(0xffffffffu, t_lane, rr);
          const float p0 = angle(tf, fh0, fl0), p1 = angle(tf, fh1, fl1);
          rotate_store(rr, rs, __cosf(p0), __sinf(p0), __cosf(p1), __sinf(p1));
        }
      }
      __syncwarp();
    }
  } else {
    const int hv = (col0 - ep.qk_cols) >> 7;
    const bool mix = ep.ve != nullptr;
    const bf16* ve_head = mix ? reinterpret_cast<const bf16*>(ep.ve) + (size_t)hv * 128 : nullptr;
    const int q = lane >> 3, c4 = lane & 7;  // lane -> (row within a group of 4, column quad)
    // value-embedding row offsets of this lane's rows 4 i + q
    const uint32_t vrow_lane = (uint32_t)tok * (uint32_t)ep.n_kv_head * 128u;
    uint32_t vr[8];
    float gr[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      vr[i] = __shfl_sync(0xffffffffu, vrow_lane, 4 * i + q);
      gr[i] = __shfl_sync(0xffffffffu, gate, 4 * i + q);
    }
    // chunk c + 1's TMEM columns and value-embedding entries are requested
    // before chunk c is mixed and stored
    uint32_t u[32];
    uint2 e[8];
    ptx::tmem_ld32(taddr, u);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      e[i] = mix ? __ldg(reinterpret_cast<const uint2*>(ve_head + vr[i] + 4 * c4)) : make_uint2(0u, 0u);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      ptx::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) stage[lane * 33 + i] = __uint_as_float(u[i]) * rscale;
      __syncwarp();
      uint2 en[8];
      if (c < 3) {
        ptx::tmem_ld32(taddr + (uint32_t)(32 * (c + 1)), u);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          en[i] = mix ? __ldg(reinterpret_cast<const uint2*>(ve_head + vr[i] + 32 * (c + 1) + 4 * c4))
                      : make_uint2(0u, 0u);
      }
      const int n = c * 32 + 4 * c4;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = 4 * i + q;
        const float* sr = stage + rr * 33 + 4 * c4;
        if (m0 + rr < a.M) {
          const float2 e01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e[i].x));
          const float2 e23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e[i].y));
          const __nv_bfloat162 b0 = __floats2bfloat162_rn(fmaf(gr[i], e01.x, sr[0]), fmaf(gr[i], e01.y, sr[1]));
          const __nv_bfloat162 b1 = __floats2bfloat162_rn(fmaf(gr[i], e23.x, sr[2]), fmaf(gr[i], e23.y, sr[3]));
          *reinterpret_cast<uint2*>(out + (size_t)(m0 + rr) * ep.ldo + n) =
              make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
        }
      }
      __syncwarp();
      if (c < 3) {
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] = en[i];
      }
    }
  }
}


// Producers of the fused norm's input (EPI_RESID / EPI_BLOCK_END) store each
// row's sum of squares over the warp's c_cnt columns [n_lo, n_lo + c_cnt) in
// slot n_lo / c_cnt of the row's ss_parts = N / c_cnt slots (lane (q, 0)
// holds the sums of rows 4 i + q).
__device__ __forceinline__ void store_row_ss(const EpiParams& ep, const TcArgs& a, int row0, int n_lo, int c_cnt,
                                             int lane, const float (&ssr)[8]) {
  if (ep.ss_out != nullptr && (lane & 7) == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int mr = row0 + 4 * i + (lane >> 3);
      if (mr < a.M) ep.ss_out[(size_t)mr * ep.ss_parts + n_lo / c_cnt] = ssr[i];
    }
  }
}

template <int BN, int MODE>
__device__ __forceinline__ RowPre epilogue_pre(const EpiParams& ep, const TcArgs& a, int mb, int nb, int g,
                                               int c_lo, int lane) {
  const int m = mb * kBM + g * 32 + lane;
  const int n_lo = nb * BN + c_lo;
  RowPre p{1.f, 0.f, -1, 0, 0.f};
  if (m >= a.M) return p;
  if constexpr (MODE == EPI_QKV || MODE == EPI_RELU2 || MODE == EPI_CE || MODE == EPI_DZ) {
    if (ep.ss_in != nullptr) {
      const float* sp = ep.ss_in + (size_t)m * ep.ss_in_parts;
      float t = 0.f;
#pragma unroll 4
      for (int j = 0; j < ep.ss_in_parts; ++j) t += sp[j];
      p.rscale = 1.0f / sqrtf(t * ep.inv_c + ep.eps);
    }
  }
  if constexpr (MODE == EPI_QKV) {
    if (n_lo % 128 == 0 && n_lo >= ep.qk_cols && n_lo < a.N && ep.ve != nullptr) {
      const int hv = (n_lo - ep.qk_cols) >> 7;
      int tok = ep.tokens[m];
      tok = min(max(tok, 0), ep.vocab - 1);
      p.tok = tok;
      const char* row = reinterpret_cast<const char*>(reinterpret_cast<const bf16*>(ep.ve) +
                                                      ((size_t)tok * ep.n_kv_head + hv) * 128);
      ptx::prefetch_l2(row);
      ptx::prefetch_l2(row + 128);
      if (ep.gate != nullptr) {
        p.gate = ep.gate[(size_t)m * ep.n_kv_head + hv];
      } else {
        // gate from the normalised block input: rscale * x[m, :gate_c]
        const float* xr = ep.x + (size_t)m * ep.ldx;
        const float* wg = ep.gate_w + (size_t)hv * ep.gate_c;
        float d = 0.f;
#pragma unroll 4
        for (int c = 0; c < ep.gate_c; ++c) d = fmaf(xr[c], wg[c], d);
        p.gate = ep.gate_scale / (1.0f + __expf(-p.rscale * d));
      }
    }
  } else if constexpr (MODE == EPI_CE || MODE == EPI_DZ) {
    int y = ep.targets[m];
    if (y != -1) y = min(max(y, 0), ep.vocab - 1);  // out-of-range ids are flagged by the combine
    p.y = y;
    if constexpr (MODE == EPI_DZ) p.lse = ep.lse[m];
  }
  return p;
}

// Epilogue work of one warp on one tile: rows g*32 .. g*32+31 of the tile
// (its TMEM lane quarter) and the columns [c_lo, c_lo + c_cnt) (a multiple
// of 32; the two warps of a lane quarter split the tile's columns).
template <int BN, int MODE>
__device__ __forceinline__ void epilogue_tile(const EpiParams& ep, const TcArgs& a, uint32_t taddr, int mb,
                                              int nb, int g, int c_lo, int c_cnt, int lane, float* stage,
                                              const RowPre& pre) {
  const int row = g * 32 + lane;
  const int m = mb * kBM + row;
  const int n_lo = nb * BN + c_lo;
  const float rscale = pre.rscale;  // fused RMSNorm of the A operand: 1 / rms of this thread's row
  if constexpr (MODE == EPI_QKV) {
    // one head (128 columns) per warp when BN = 256; with BN = 128 the first half does it
    if (c_lo % 128 == 0 && n_lo < a.N)
      epi_qkv_head(ep, a, stage, taddr + (uint32_t)c_lo, mb * kBM + g * 32, lane, n_lo, rscale, pre.gate, pre.tok);
  } else if constexpr (MODE == EPI_CE) {
    const int y = pre.y;
    // zhat = c tanh(z/c) = c - 2c / (e^{2z/c} + 1); exp(zhat - c) = 2^(-2c log2(e) / (e^{2z/c} + 1))
    const float k1 = 2.0f * 1.4426950408889634f / ep.cap;
    const float k2 = -2.0f * ep.cap * 1.4426950408889634f;
    const float c2 = -2.0f * ep.cap;
    float sum = 0.f, tgt = 0.f;
#pragma unroll 1
    for (int c = 0; c < c_cnt; c += 32) {
      uint32_t r[32];
      ptx::tmem_ld32(taddr + (uint32_t)(c_lo + c), r);
      ptx::tmem_ld_wait();
      const int n = n_lo + c;
      float zh[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float q = ptx::rcp(ptx::ex2(__uint_as_float(r[i]) * (rscale * k1)) + 1.0f);
        zh[i] = fmaf(c2, q, ep.cap);
        const float p = ptx::ex2(k2 * q);
        sum += (n + i < ep.vocab) ? p : 0.f;
        tgt = (n + i == y) ? zh[i] : tgt;
      }
      if (ep.logits != nullptr && m < a.M) {
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
    }
    if (m < a.M) {
      ep.ce_sum[(size_t)m * ep.ce_tiles + nb * 2 + (2 * c_lo) / BN] = sum;
      if (y >= n_lo && y < n_lo + c_cnt) ep.ce_tgt[m] = tgt;
    }
  } else if constexpr (MODE == EPI_DZ || MODE == EPI_F32) {
    const float ginv = MODE == EPI_DZ ? *ep.inv_count : 0.f;
    uint32_t r[32];
    ptx::tmem_ld32(taddr + (uint32_t)c_lo, r);
#pragma unroll 1
    for (int c = 0; c < c_cnt; c += 32) {
      ptx::tmem_ld_wait();
      uint32_t rc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) rc[i] = r[i];
      if (c + 32 < c_cnt) ptx::tmem_ld32(taddr + (uint32_t)(c_lo + c + 32), r);
      epi_bwd_chunk<MODE>(ep, a, stage, mb * kBM + g * 32, n_lo + c, rc, lane, pre, ginv);
    }
  } else if constexpr (MODE == EPI_RESID) {
    float ssr[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int row0 = mb * kBM + g * 32;
    uint32_t r[32];
    float4 xv[8];
    ptx::tmem_ld32(taddr + (uint32_t)c_lo, r);
    resid_load(ep, a, row0, n_lo, lane, xv);
#pragma unroll 1
    for (int c = 0; c < c_cnt; c += 32) {
      ptx::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) stage[lane * 33 + i] = __uint_as_float(r[i]);
      __syncwarp();
      float4 xn[8];
      if (c + 32 < c_cnt) {
        ptx::tmem_ld32(taddr + (uint32_t)(c_lo + c + 32), r);
        resid_load(ep, a, row0, n_lo + c + 32, lane, xn);
      }
      resid_apply(ep, a, stage, row0, n_lo + c, lane, xv, ssr);
      __syncwarp();
      if (c + 32 < c_cnt) {
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[i] = xn[i];
      }
    }
    store_row_ss(ep, a, row0, n_lo, c_cnt, lane, ssr);
  } else {
    float ssr[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // chunk c + 1's TMEM columns are requested before chunk c is processed
    uint32_t r[32];
    ptx::tmem_ld32(taddr + (uint32_t)c_lo, r);
#pragma unroll 1
    for (int c = 0; c < c_cnt; c += 32) {
      ptx::tmem_ld_wait();
      uint32_t rc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) rc[i] = r[i];
      if (c + 32 < c_cnt) ptx::tmem_ld32(taddr + (uint32_t)(c_lo + c + 32), r);
      if constexpr (MODE == EPI_BLOCK_END) {
        epi_resid_chunk(ep, a, stage, mb * kBM + g * 32, n_lo + c, rc, lane, ssr);
      } else {
        epi_store_chunk(ep, a, stage, mb * kBM + g * 32, n_lo + c, rc, lane, MODE == EPI_RELU2, rscale);
      }
    }
    if constexpr (MODE == EPI_BLOCK_END) store_row_ss(ep, a, mb * kBM + g * 32, n_lo, c_cnt, lane, ssr);

  }
}

// AMN / BMN = 1: that operand is stored MN-major (the transpose of the
// K-major layout), loaded as 64 x 64 boxes (64 MN elements = one 128-byte
// swizzled row, 64 k rows) placed 8 KB apart, and read by the MMA through an
// MN-major descriptor (leading offset 8 KB between 64-wide MN blocks, a
// 16-row k step = 2 KB).
template <int BN, int MODE, int AMN = 0, int BMN = 0>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const TcArgs a, const EpiParams ep) {
  using Cf = TcCfg<BN>;
  constexpr int S = Cf::STAGES;
  pdl_launch_dependents();
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
      ptx::mbar_init(tempty(i), kEpiWarps);
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
  const int nk = (a.K + kBK - 1) / kBK;  // k beyond K reads zeros (tensor-map bounds)
  pdl_wait();  // the operands and the epilogue's inputs come from earlier kernels

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
          if constexpr (AMN) {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              ptx::tma_load_2d(sA(stage) + j * 8192, &tmA, full(stage), mb * kBM + 64 * j, kb * kBK);
          } else {
            ptx::tma_load_2d(sA(stage), &tmA, full(stage), kb * kBK, mb * kBM);
          }
          if constexpr (BMN) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              ptx::tma_load_2d(sB(stage) + j * 8192, &tmB, full(stage), nb * BN + 64 * j, kb * kBK);
          } else {
            ptx::tma_load_2d(sB(stage), &tmB, full(stage), kb * kBK, nb * BN);
          }
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
      constexpr uint32_t idesc = ptx::idesc_bf16(kBM, BN, AMN, BMN);
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
          const uint64_t da = AMN ? ptx::desc_mnmajor_sw128(sA(stage), 8192) : ptx::desc_kmajor_sw128(sA(stage));
          const uint64_t db = BMN ? ptx::desc_mnmajor_sw128(sB(stage), 8192) : ptx::desc_kmajor_sw128(sB(stage));
          // a k step of 16 is 32 bytes along a K-major row, 16 rows (2 KB) of an MN-major box
          constexpr uint64_t ka = AMN ? (2048 >> 4) : 2, kb16 = BMN ? (2048 >> 4) : 2;
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k)
            ptx::mma_bf16_ss(d, da + ka * k, db + kb16 * k, idesc, (kb | k) != 0 ? 1u : 0u);
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
    // ---------------- epilogue (warps 2 .. 2 + kEpiWarps - 1) ----------------
    // two warps per TMEM lane quarter, each taking half of the tile's columns
    const int ew = warp - 2;
    const int g = warp & 3;
    const int half = ew >> 2;
    const int c_lo = half * (BN / 2), c_cnt = BN / 2;
    float* stage = epi_stage + ew * Cf::STAGE_FLOATS;
    int acc = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      const int mb = tile % a.tiles_m, nb = tile / a.tiles_m;
      const RowPre pre = epilogue_pre<BN, MODE>(ep, a, mb, nb, g, c_lo, lane);
      if (*abort_flag || !ptx::mbar_wait(tfull(acc), aph, a.status)) {
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(g * 32) << 16) + (uint32_t)(acc * BN);
      epilogue_tile<BN, MODE>(ep, a, taddr, mb, nb, g, c_lo, c_cnt, lane, stage, pre);
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

// ---------------------------------------------------------------------------
// CTA-pair variant (cluster of 2, tcgen05 cta_group::2): a 256 x 256 output
// tile per pair.  Each CTA loads its own 128 rows of A and its own 128 rows
// (half) of B per k-slice, so a CTA moves 32 KB instead of 48 KB per 128 x 256
// x 64 step; the even CTA issues M = 256 MMAs over both CTAs' shared memory
// and each CTA's TMEM receives its 128 rows.  Both CTAs' copies complete on
// the even CTA's "full" barrier; MMA completion is multicast to both CTAs'
// "empty"/"accumulator full" barriers; both CTAs' epilogues arrive on the even
// CTA's "accumulator empty" barrier.  No TMA multicast: every CTA reads its
// own operand slices.
// ---------------------------------------------------------------------------
// Pair kernel roles: warps 0..7 epilogue (two warpgroups), warp 8 TMA,
// warp 9 MMA + TMEM allocation, warps 10..11 idle.  Registers: launched at
// 168 per thread (65536 / 384); the TMA/MMA warpgroup drops to 88 and the
// epilogue warpgroups rise to 208: 2 * 128 * 208 + 128 * 88 = 64512 = 384 * 168.
constexpr int kPairThreads = 384;
constexpr int kPairWarpTma = 8, kPairWarpMma = 9;
constexpr int kPairRegsLow = 88, kPairRegsHigh = 208;
static_assert(2 * 128 * kPairRegsHigh + 128 * kPairRegsLow <= kPairThreads * 168, "register split");

// BN_: the pair tile's width.
template <int BN_>
struct PairCfg {
  static constexpr int BN = BN_;
  static constexpr int STAGES = BN == 256 ? 6 : 8;
  static constexpr int A_BYTES = kBM * kBK * 2;       // 16 KB: this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * kBK * 2;  // this CTA's BN/2 rows of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static_assert(STAGE_BYTES % 1024 == 0, "stages stay aligned to the 128-byte swizzle atom");
  static constexpr int TMEM_COLS = BN == 256 ? 512 : 256;  // two accumulators, rounded to a power of 2
  static constexpr int NBARS = 2 * STAGES + 5;
  static constexpr int STAGE_FLOATS = 32 * 33;
  static constexpr int EPI_BYTES = kEpiWarps * STAGE_FLOATS * 4;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256 + EPI_BYTES;
};

template <int MODE, int BN_ = 256>
__global__ void __launch_bounds__(kPairThreads, 1)
    k_gemm_tc2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const TcArgs a, const EpiParams ep) {
  using Cf = PairCfg<BN_>;
  constexpr int BN = Cf::BN;
  constexpr int S = Cf::STAGES;
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cf::STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cf::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_stage = reinterpret_cast<float*>(smem + S * Cf::STAGE_BYTES + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
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
      ptx::mbar_init(tempty(i), 2 * kEpiWarps);  // both CTAs' epilogue warps (used on the even CTA)
    }
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
  }
  if (warp == kPairWarpMma) {
    ptx::tmem_alloc2(ptx::smem_u32(tmem_slot), Cf::TMEM_COLS);
    ptx::tmem_relinquish2();
    ptx::tc_fence_before();
  }
  // barriers of both CTAs are initialised before any cross-CTA signal
  ptx::cluster_sync_all();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nk = a.K / kBK;
  pdl_wait();  // the operands and the epilogue's inputs come from earlier kernels
  const int tiles_mp = (a.M + 2 * kBM - 1) / (2 * kBM);
  const int num_pt = tiles_mp * a.tiles_n;
  const int cid = (int)ptx::cluster_id_x(), ncl = (int)ptx::nclusters_x();
  const PairSched sched = make_sched(a, num_pt, nk, cid, ncl);

  if (warp >= 8) {
    ptx::setmaxnreg_dec<kPairRegsLow>();
    if (warp == kPairWarpTma) {
    if (ptx::elect_one()) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t ph = 0, issued = 0, par = 0;
      for (int j = 0; j < sched.njobs; ++j) {
        int pt, kb_lo, kb_hi, kind;
        job_at(sched, j, pt, kb_lo, kb_hi, kind);
        int mbp, nb;
        pair_tile(a, pt, tiles_mp, mbp, nb);
        kb_hi = min(kb_hi, tile_kb_end(a, nb, BN, nk));
        bool ok = true;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (*abort_flag || !ptx::mbar_wait_cluster(empty(stage), ph ^ 1, a.status)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (leader) ptx::mbar_arrive_expect_tx(full(stage), 2 * Cf::STAGE_BYTES);
          const uint32_t fb = ptx::mapa(full(stage), 0);
          ptx::tma_load_2d_pair(sA(stage), &tmA, fb, kb * kBK, mbp * 2 * kBM + (int)rank * kBM);
          ptx::tma_load_2d_pair(sB(stage), &tmB, fb, kb * kBK, nb * BN + (int)rank * (BN / 2));
          issued |= 1u << stage;
          par = (par & ~(1u << stage)) | (ph << stage);
          if (++stage == S) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
      // this CTA's copies have landed (and been consumed) before it may exit
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) ptx::mbar_wait_cluster(empty(s), (par >> s) & 1, a.status);
    }
  } else if (warp == kPairWarpMma) {
    if (leader && ptx::elect_one()) {
      // ---------------- MMA issuer (even CTA) ----------------
      constexpr uint32_t idesc = ptx::idesc_bf16(2 * kBM, BN);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      for (int j = 0; j < sched.njobs; ++j) {
        int pt, kb_lo, kb_hi, kind;
        job_at(sched, j, pt, kb_lo, kb_hi, kind);
        {
          int mbp, nb;
          pair_tile(a, pt, tiles_mp, mbp, nb);
          kb_hi = min(kb_hi, tile_kb_end(a, nb, BN, nk));
        }
        if (*abort_flag || !ptx::mbar_wait_cluster(tempty(acc), aph ^ 1, a.status)) {
          *abort_flag = 1;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (*abort_flag || !ptx::mbar_wait_cluster(full(stage), ph, a.status)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t da = ptx::desc_kmajor_sw128(sA(stage));
          const uint64_t db = ptx::desc_kmajor_sw128(sB(stage));
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k)
            ptx::mma_bf16_ss2(d, da + 2 * k, db + 2 * k, idesc, (kb != kb_lo || k != 0) ? 1u : 0u);
          ptx::mma_commit2_mc(empty(stage), 0x3);
          if (++stage == S) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        ptx::mma_commit2_mc(tfull(acc), 0x3);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      // all MMAs have completed before either CTA releases its TMEM
      ptx::mma_commit2(mma_done);
      ptx::mbar_wait_cluster(mma_done, 0, a.status);
    }
    }
  } else {
    ptx::setmaxnreg_inc<kPairRegsHigh>();
    // ---------------- epilogue (both CTAs, warps 0 .. kEpiWarps - 1) ----------------
    const int ew = warp;
    const int g = warp & 3;  // TMEM lane quarter
    const int half = ew >> 2;
    // the two warps of a lane quarter take the two column halves of the tile
    auto cols = [&](int, int& c_lo, int& c_cnt) {
      c_lo = half * (BN / 2);
      c_cnt = BN / 2;
    };
    float* stage = epi_stage + ew * Cf::STAGE_FLOATS;
    int acc = 0;
    uint32_t aph = 0;
    for (int j = 0; j < sched.njobs; ++j) {
      int pt, kb_lo, kb_hi, kind;
      job_at(sched, j, pt, kb_lo, kb_hi, kind);
      const bool head = kind == 1;  // k-blocks of a tile another pair finishes: write a partial
      const bool tail = kind == 2;  // finishes a tile: add the earlier pairs' partials
      int mbp, nb, c_lo, c_cnt;
      pair_tile(a, pt, tiles_mp, mbp, nb);
      cols(j, c_lo, c_cnt);
      const RowPre pre = epilogue_pre<BN, MODE>(ep, a, mbp * 2 + (int)rank, nb, g, c_lo, lane);
      if (*abort_flag || !ptx::mbar_wait_cluster(tfull(acc), aph, a.status)) {
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(g * 32) << 16) + (uint32_t)(acc * BN);
      // this CTA's 128 x 256 partial: column c, row r at slot * 32768 + c * 128 + r
      const int row = g * 32 + lane;
      const int col0 = half * (BN / 2);
      if (head) {
        float* slot = a.sk_ws + (size_t)(cid * 2 + (int)rank) * (128 * BN);
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(taddr + (uint32_t)(col0 + c), r);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) slot[(size_t)(col0 + c + i) * 128 + row] = __uint_as_float(r[i]);
        }
        // all epilogue warps of this CTA have written their part before the flag
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory");
        if (warp == 0 && lane == 0) {
          __threadfence();
          ptx::st_release_gpu(a.sk_flags + cid * 2 + (int)rank, a.sk_gen);
        }
      } else {
        if (tail) {
          // add the partials of the pairs before this one that hold the
          // tile's earlier k-blocks (same CTA rank) into TMEM
          const long long U = (long long)(num_pt - sched.tail_pt0) * nk;
          const int c_first = first_contributor(sched, U, (long long)(pt - sched.tail_pt0));
#pragma unroll 1
          for (int cp = c_first; cp < cid; ++cp) {
            if (U * (cp + 1) / ncl == U * cp / ncl) continue;  // pair cp has no tail units
            const unsigned* flag = a.sk_flags + cp * 2 + (int)rank;
            bool ready = ptx::ld_acquire_gpu(flag) == a.sk_expect;
            if (!ready) {
              const uint64_t t0 = ptx::globaltimer();
              while (!(ready = ptx::ld_acquire_gpu(flag) == a.sk_expect))
                if (ptx::globaltimer() - t0 > a.sk_wait_ns) break;
            }
            if (!__all_sync(0xffffffffu, ready)) {
              atomicOr(a.status, kStatusTimeout);
              *abort_flag = 1;
              break;
            }
            const float* slot = a.sk_ws + (size_t)(cp * 2 + (int)rank) * (128 * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 2; c += 32) {
              uint32_t r[32];
              ptx::tmem_ld32(taddr + (uint32_t)(col0 + c), r);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i)
                r[i] = __float_as_uint(__uint_as_float(r[i]) + slot[(size_t)(col0 + c + i) * 128 + row]);
              ptx::tmem_st32(taddr + (uint32_t)(col0 + c), r);
            }
            ptx::tmem_st_wait();
          }
        }
        epilogue_tile<BN, MODE>(ep, a, taddr, mbp * 2 + (int)rank, nb, g, c_lo, c_cnt, lane, stage, pre);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa(tempty(acc), 0));
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }
  __syncthreads();
  ptx::cluster_sync_all();
  if (warp == kPairWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc2(tmem, Cf::TMEM_COLS);
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

template <int BN, int MODE>
bool launch_mode(const CUtensorMap& ta, const CUtensorMap& tb, const TcArgs& a, const EpiParams& ep, int grid,
                 cudaStream_t st) {
  if (!smem_optin(k_gemm_tc<BN, MODE>, TcCfg<BN>::SMEM)) return false;
  return launch_pdl(k_gemm_tc<BN, MODE>, dim3(grid), dim3(kThreads), TcCfg<BN>::SMEM, st, 1, ta, tb, a, ep) ==
         cudaSuccess;
}

template <int MODE, int AMN, int BMN>
bool launch_layout_mode(const CUtensorMap& ta, const CUtensorMap& tb, const TcArgs& a, const EpiParams& ep, int grid,
                        cudaStream_t st) {
  if (!smem_optin(k_gemm_tc<256, MODE, AMN, BMN>, TcCfg<256>::SMEM)) return false;
  return launch_pdl(k_gemm_tc<256, MODE, AMN, BMN>, dim3(grid), dim3(kThreads), TcCfg<256>::SMEM, st, 1, ta, tb, a,
                    ep) == cudaSuccess;
}

template <int MODE, int BN = 256>
bool launch_pair_mode(const CUtensorMap& ta, const CUtensorMap& tb, const TcArgs& a, const EpiParams& ep,
                      int nclusters, cudaStream_t st) {
  if (!smem_optin(k_gemm_tc2<MODE, BN>, PairCfg<BN>::SMEM)) return false;
  return launch_pdl(k_gemm_tc2<MODE, BN>, dim3(2 * nclusters), dim3(kPairThreads), PairCfg<BN>::SMEM, st, 2, ta, tb,
                    a, ep) == cudaSuccess;
}

bool launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const TcArgs& a, const EpiParams& ep, int nclusters,
                 cudaStream_t st, int bn) {
  if (bn != 256) return false;
  switch (ep.mode) {
    case EPI_STORE: return launch_pair_mode<EPI_STORE>(ta, tb, a, ep, nclusters, st);
    case EPI_RELU2: return launch_pair_mode<EPI_RELU2>(ta, tb, a, ep, nclusters, st);
    case EPI_RESID: return launch_pair_mode<EPI_RESID>(ta, tb, a, ep, nclusters, st);
    case EPI_BLOCK_END: return launch_pair_mode<EPI_BLOCK_END>(ta, tb, a, ep, nclusters, st);
    case EPI_CE: return launch_pair_mode<EPI_CE>(ta, tb, a, ep, nclusters, st);
    case EPI_QKV: return launch_pair_mode<EPI_QKV>(ta, tb, a, ep, nclusters, st);
    case EPI_F32: return launch_pair_mode<EPI_F32>(ta, tb, a, ep, nclusters, st);
    default: return false;
  }
}

template <int BN>
bool launch_bn(const CUtensorMap& ta, const CUtensorMap& tb, const TcArgs& a, const EpiParams& ep, int grid,
               cudaStream_t st) {
  switch (ep.mode) {
    case EPI_STORE: return launch_mode<BN, EPI_STORE>(ta, tb, a, ep, grid, st);
    case EPI_RELU2: return launch_mode<BN, EPI_RELU2>(ta, tb, a, ep, grid, st);
    case EPI_RESID: return launch_mode<BN, EPI_RESID>(ta, tb, a, ep, grid, st);
    case EPI_BLOCK_END: return launch_mode<BN, EPI_BLOCK_END>(ta, tb, a, ep, grid, st);
    case EPI_CE: return launch_mode<BN, EPI_CE>(ta, tb, a, ep, grid, st);
    case EPI_QKV: return launch_mode<BN, EPI_QKV>(ta, tb, a, ep, grid, st);
    default: return false;
  }
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

bool launch_gemm_tc_layout(const bf16* A, int lda, int a_mn, const bf16* Bm, int ldb, int b_mn, int M, int N, int K,
                           const EpiParams& ep, int* status, int num_sms, cudaStream_t st) {
  constexpr int BN = 256;
  CUtensorMap ta, tb;
  // K-major: [rows, K] with boxes of 64 k x rows; MN-major: [K, MN] with 64 x 64 boxes
  if (!(a_mn ? make_tmap_2d(&ta, A, K, M, lda, 64, 64) : make_tmap_2d(&ta, A, M, K, lda, kBM, kBK))) return false;
  if (!(b_mn ? make_tmap_2d(&tb, Bm, K, N, ldb, 64, 64) : make_tmap_2d(&tb, Bm, N, K, ldb, BN, kBK))) return false;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = (M + kBM - 1) / kBM;
  a.tiles_n = (N + BN - 1) / BN;
  a.num_tiles = a.tiles_m * a.tiles_n;
  a.status = status;
  a.sk_wait_ns = kWaitLimitNs;
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  LaunchScope scope_(KK_GEMM_TC_BWD, st);
  if (ep.mode == EPI_DZ && !a_mn && !b_mn) return launch_layout_mode<EPI_DZ, 0, 0>(ta, tb, a, ep, grid, st);
  if (ep.mode == EPI_F32 && !a_mn && b_mn) return launch_layout_mode<EPI_F32, 0, 1>(ta, tb, a, ep, grid, st);
  if (ep.mode == EPI_F32 && a_mn && b_mn) return launch_layout_mode<EPI_F32, 1, 1>(ta, tb, a, ep, grid, st);
  return false;
}

bool launch_gemm_tc(const bf16* A, int lda, const bf16* Bm, int ldb, int M, int N, int K,
                    const EpiParams& ep, int* status, int num_sms, cudaStream_t st, bool pair,
                    const StreamK* sk, const GemmKLimit* kl) {
  const int BN = gemm_tc_bn(N);
  if (pair && BN == 256 && num_sms >= 2) {
    // CTA pairs: each CTA loads 128 rows of A and 128 rows of B per k-slice.
    // (256 x 96 tiles would quantise N = 1536 into 6.92 waves instead of 2.59
    // run as 3, but each CTA then streams 22 KB of operands per 1.6 MFLOP of
    // MMA, more than L2 delivers to 148 SMs at once: measured 13.9 ms per d24
    // step against 12.3 ms with 256 x 256 tiles.)
    const int bnp = 256;
    CUtensorMap ta, tb;
    if (!make_tmap_2d(&ta, A, M, K, lda, kBM, kBK)) return false;
    if (!make_tmap_2d(&tb, Bm, N, K, ldb, bnp / 2, kBK)) return false;
    TcArgs a;
    memset(&a, 0, sizeof(a));
    a.M = M;
    a.N = N;
    a.K = K;
    a.tiles_m = (M + kBM - 1) / kBM;
    a.tiles_n = N / bnp;
    a.num_tiles = a.tiles_m * a.tiles_n;
    a.n_fastest = ep.mode != EPI_CE;
    a.status = status;
    const int num_pt = ((M + 2 * kBM - 1) / (2 * kBM)) * a.tiles_n;
    const int ncl = num_pt < num_sms / 2 ? num_pt : num_sms / 2;
    // stream-K when every pair's share spans at least two tiles and the
    // buffers for the pairs' partial sums are there
    const int nk = K / kBK;
    a.streamk = 0;
    a.sk_ws = nullptr;
    a.sk_flags = nullptr;
    a.sk_gen = 0;
    a.sk_expect = 0;
    a.sk_wait_ns = kWaitLimitNs;
    // (and when the partial wave is at least a quarter full, so that a tile is
    // cut among a few pairs only)
    if (sk != nullptr && sk->ws != nullptr && ncl <= sk->max_pairs && ep.mode == EPI_BLOCK_END && nk >= 1 &&
        num_pt >= ncl && num_pt % ncl != 0 && 4 * (num_pt % ncl) >= ncl) {
      a.streamk = 1;
      a.sk_ws = sk->ws;
      a.sk_flags = sk->flags;
      a.sk_gen = sk->gen;
      unsigned skew = 0;
      flag_wait_test(&a.sk_wait_ns, &skew);
      a.sk_expect = sk->gen + skew;
    }
    a.kl_k = 0;
    if (kl != nullptr && !a.streamk) {
      a.kl_k = kl->out.k;
      for (int i = 0; i < kMaxPrefixBlocks; ++i) {
        a.kl_out_end[i] = i < kl->out.k ? kl->out.end[i] : 0;
        a.kl_in_end[i] = i < kl->in.k ? kl->in.end[i] : 0;
      }
    }
    LaunchScope scope_(KK_GEMM_TC, st);
    return launch_pair(ta, tb, a, ep, ncl, st, bnp);
  }
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, M, K, lda, kBM, kBK)) return false;
  if (!make_tmap_2d(&tb, Bm, N, K, ldb, BN, kBK)) return false;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = (M + kBM - 1) / kBM;
  a.tiles_n = (N + BN - 1) / BN;
  a.num_tiles = a.tiles_m * a.tiles_n;
  a.n_fastest = 0;  // unused by the single-CTA kernel
  a.status = status;
  a.streamk = 0;
  a.sk_ws = nullptr;
  a.sk_flags = nullptr;
  a.sk_gen = 0;
  a.sk_expect = 0;
  a.sk_wait_ns = kWaitLimitNs;
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  LaunchScope scope_(KK_GEMM_TC, st);
  return BN == 256 ? launch_bn<256>(ta, tb, a, ep, grid, st) : launch_bn<128>(ta, tb, a, ep, grid, st);
}

}  // namespace nc
