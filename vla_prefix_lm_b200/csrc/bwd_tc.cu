// bwd_tc.cu -- gradient of the joint prefill (dq, dk, dv) on tcgen05 tensor
// cores: bf16 inputs, one KV head, head_dim 256.  The training step runs the
// joint forward under gradient ("VLA 代码精读 - OpenPI & StarVLA", 1.5
// Pi0.compute_loss); the pages print no backward, so this is the plain
// derivative of the forward:
//     P = exp(scale * Q K^T - lse)  (the forward's lse; 0 where masked)
//     dP = dO V^T,   D = rowsum(dO * O),   dS = P * (dP - D)
//     dV = P^T dO,   dK = scale * dS^T Q,   dQ = scale * dS K
// over the flattened (token, head) rows of each batch element; with one KV
// head every row reads the same keys.
//
// Tensor memory holds 512 fp32 columns per SM.  At head_dim 256 the dK and dV
// accumulators of one 128-key tile fill it, leaving no room for the score
// tiles a single key-stationary pass would recompute; shared memory likewise
// cannot double-buffer K and V beside a resident Q and dO.  The gradient is
// therefore split into three passes that together run the five contractions
// once each, every one on tcgen05 pair MMAs (cta_group::2, M = 256 rows over a
// cluster of two CTAs):
//
//   score pass  query-major: S = Q K^T and dP = dO V^T on 128-key tiles into
//               TMEM (N = 128 pair MMAs in TS form: the row tile's Q and dO
//               sit in TMEM as the A operand, 256 of the 512 columns, copied
//               in by the row warps when the row tile changes; S and dP take
//               the other 256, one buffer each, freed separately so that the
//               next tile's S MMAs run while dP is read); one thread per row
//               and 32 keys forms P and dS in fp32 and writes both as bf16 to
//               the caller's workspace [B, rows, Skp] (Skp = S rounded up to 64).
//               Persistent: each SM pair takes an equal, contiguous run of the
//               (batch, 256-row tile, key tile) sequence; shared memory holds
//               a two-stage K/V ring and the P/dS store stages.
//   dK/dV pass  key-major, per 256-key group: dV += P^T dO and dK += dS^T Q
//               over 64-row steps, P^T and dS^T read MN-major from the
//               workspace; small problems split the rows into chunks whose
//               partial sums a reduction kernel adds in a fixed order.
//   dQ pass     per 256-row tile: dQ += dS K over the same 64-key tiles.
//               Persistent, with two TMEM accumulators so that one tile's
//               epilogue overlaps the next tile's MMAs.
//
// Tiles are skipped by the forward's rule: a 256-key group is visited by a
// 256-row tile unless no row of it sees any key of the group (block index,
// expert <- FAST, padding).  The score pass writes both 128-key tiles of a
// visited group (exact zeros where masked), so the dK/dV pass, which reads
// whole groups, never reads an unwritten block.  Rows go to global memory
// through a per-warp shared-memory transpose, so every store instruction
// writes whole 128-byte lines.  Everything is deterministic (no atomics).
// Every wait is bounded (DevCtl) and a timeout is reported in the status word.
#include <cfloat>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kT = 192;          // warp 0 TMA, warp 1 TMEM + MMA issue, warps 2..5 rows
constexpr int kT1 = 576;         // score pass: warps 2..17 rows, four per TMEM lane quarter
constexpr int kRows = 128;       // rows per CTA (256 per pair)
constexpr int kD = 256;
constexpr int kKT = 64;          // keys per score tile (32 per CTA)
constexpr int kSup = 256;        // keys per group (4 score tiles; one dK/dV tile)
constexpr int kSmemLimit = 232448;
constexpr int kMaxTiles128 = (kMaxTokens + 127) / 128 + 1;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory operand sizes (bf16, 128-byte swizzled [rows x 64] blocks).
constexpr int kKT1 = 128;        // keys per score-pass tile (64 per CTA)
constexpr int kItem64 = 64 * kD * 2;           // [64 x 256]    32 KB (this CTA's keys of a score tile)
constexpr int kHalf64 = 64 * 128 * 2;          // [64 x 128]    16 KB (64 rows/keys x this CTA's d-half)
constexpr int kDsTile = kRows * 64 * 2;        // [128 x 64]    16 KB (dS rows of a 64-key tile)
constexpr int kWarpStage = 32 * 128;           // 4 KB per row warp: 32 rows x 128 B transpose

constexpr int kNS2 = 3, kNS3 = 4;              // ring stages of the dK/dV and dQ passes
constexpr int kStage1 = 2 * kItem64;           // K, V items
constexpr int kNS1 = 2;                        // ring stages of the score pass
constexpr int kBox1 = 32 * 64;                 // 2 KB per score row warp: one 32 x 32 bf16 box
constexpr int kStage2 = 4 * kHalf64;           // P^T, dS^T, dO half, Q half
constexpr int kStage3 = kDsTile + kHalf64;     // dS tile, K half
constexpr int kOps1 = kNS1 * kStage1 + 16 * kBox1;             // 160 KB
constexpr int kOps2 = kNS2 * kStage2;                        // 192 KB
constexpr int kOps3 = kNS3 * kStage3 + 4 * kWarpStage;       // 144 KB

constexpr uint32_t kIdescScore = idesc_bf16_f32(2 * kRows, kKT1, false, false);
constexpr uint32_t kIdescKV = idesc_bf16_f32(2 * kRows, kD, true, true);
constexpr uint32_t kIdescQ = idesc_bf16_f32(2 * kRows, kD, false, true);

struct __align__(8) Ctl {
  uint64_t full[4];       // leader: a ring stage of both CTAs landed
  uint64_t empty[4];      // each CTA: its stage may be refilled
  uint64_t qd_full;       // leader (score pass): the pair's 32 row warps put Q and dO in TMEM
  uint64_t s_full[2];     // each CTA (score pass): S [0] / dP [1] of a tile in TMEM
  uint64_t s_free[2];     // leader (score pass): the pair's 32 row warps read S / dP
  uint64_t done[2];       // each CTA: an accumulator is final
  uint64_t acc_free[2];   // leader (dQ pass): the pair's 8 row warps read an accumulator
  uint64_t drain;         // leader: every MMA issued has completed
  uint32_t tmem_base;
  int abort;
  int scan[kT1 / 32];
  uint16_t cs_first[kMaxTiles128];
  uint16_t cs_last[kMaxTiles128];
  uint8_t flags[kMaxTiles128];
};

__host__ __device__ constexpr int ctl_bytes() { return ((int)sizeof(Ctl) + 127) / 128 * 128; }
__host__ __device__ constexpr int pad128(int n) { return (n + 127) / 128 * 128; }
// Operands, control block, `extra` bytes (rounded to 128), per-token codes.
__host__ __device__ constexpr int smem_need(int ops, int S, int extra) {
  return ops + ctl_bytes() + pad128(extra) + pad128(S) * 2;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* abort,
                                              const DevCtl& ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*(volatile int*)abort) return false;
    if ((unsigned long long)(clock64() - t0) > ctl.wait_limit) {
      record_status(ctl, kStatusTimeout);
      *(volatile int*)abort = 1;
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Ctl& c,
                                          const DevCtl& ctl) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, &c.abort, ctl));
}

__device__ __forceinline__ void commit_both(uint64_t* bar) {
  umma_commit_pair(mapa_shared(smem_u32(bar), 0));
  umma_commit_pair(mapa_shared(smem_u32(bar), 1));
}

// Whether a 256-row tile whose last token has block index csq1 (all of whose
// tokens are expert or padding if all_e) may see a key of the 256-key group
// ks.  False only when no pair of the two can be visible: every key's block
// index is above every row's, the rows are experts and the keys FAST, or the
// keys are all padding.
__device__ __forceinline__ bool group_visible(const Ctl& c, uint32_t csq1, bool all_e, int ks,
                                              int S) {
  const int t0 = 2 * ks;
  const int n128 = (S + 127) / 128;
  if (t0 >= n128) return false;
  if (c.cs_first[t0] > csq1) return false;
  const bool two = t0 + 1 < n128;
  const uint32_t f0 = c.flags[t0], f1 = two ? c.flags[t0 + 1] : 0xFu;
  if ((f0 & 8u) && (f1 & 8u)) return false;                 // all padding
  if (all_e && (f0 & 2u) && (f1 & 2u)) return false;        // experts vs FAST
  return true;
}

// The visited 64-key tile after `kt` (-1: the first) of a row tile, or -1.
__device__ __forceinline__ int next_tile(const Ctl& c, uint32_t csq1, bool all_e, int kt, int S,
                                         int n_kt) {
  int t = kt + 1;
  while (t < n_kt) {
    if ((t & 3) != 0) return t;                 // the rest of a visited group
    if (group_visible(c, csq1, all_e, t >> 2, S)) return t;
    t += 4;
  }
  return -1;
}

// 1 if every token of [tq0, tq1] is an expert (or padding) token.
__device__ __forceinline__ bool tokens_all_expert_serial(const uint16_t* codes, int tq0, int tq1) {
  for (int t = tq0; t <= tq1; ++t)
    if (((codes[t] >> 1) & 1) == 0) return false;
  return true;
}

// Warp-collective store of 32 rows x 128 bytes: lane t holds row t's bytes in
// v[0..7] (16 bytes each) and row t goes to seg(t).  The rows pass through a
// 4 KB shared-memory transpose (16-byte chunks XOR-swizzled by row, so both
// directions are free of bank conflicts); each store instruction then writes
// four whole rows (four 128-byte lines) instead of 32 scattered pieces.  Rows
// whose bit in `valid` is clear are not written.
template <class SegFn>
__device__ __forceinline__ void store_rows128(uint8_t* stage, const uint4 (&v)[8], uint32_t valid,
                                              int lane, SegFn seg) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(stage + lane * 128 + ((j ^ (lane & 7)) << 4)) = v[j];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + (lane >> 3), j = lane & 7;
    const uint4 x = *reinterpret_cast<const uint4*>(stage + r * 128 + ((j ^ (r & 7)) << 4));
    if ((valid >> r) & 1u) *reinterpret_cast<uint4*>(seg(r) + 16 * j) = x;
  }
  __syncwarp();
}

// Warp-collective: 32 TMEM lanes (rows) x 256 fp32 columns from `taddr`,
// times `mul`, to rows row_ptr(r) (256 fp32 each, 16-byte aligned), written
// in 128-byte lines through `stage`; zeros (no TMEM read) when `zero`.
template <class RowFn>
__device__ __forceinline__ void tmem_rows_out(uint32_t taddr, float mul, uint8_t* stage,
                                              uint32_t valid, int lane, bool zero, RowFn row_ptr) {
#pragma unroll 1
  for (int cc = 0; cc < kD / 32; ++cc) {
    uint32_t o[32];
    if (!zero) {
      tmem_ld32(taddr + 32 * cc, o);
      tmem_ld_wait();
      reg_fence(o);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0u;
    }
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      v[j] = make_uint4(__float_as_uint(__uint_as_float(o[4 * j]) * mul),
                        __float_as_uint(__uint_as_float(o[4 * j + 1]) * mul),
                        __float_as_uint(__uint_as_float(o[4 * j + 2]) * mul),
                        __float_as_uint(__uint_as_float(o[4 * j + 3]) * mul));
    store_rows128(stage, v, valid, lane, [&](int r) {
      return reinterpret_cast<uint8_t*>(row_ptr(r) + 32 * cc);
    });
  }
}

// Common prologue: align the shared-memory base and check the layout fits.
// Returns nullptr (after recording PI_ERR_UNSUPPORTED) if it does not.
__device__ __forceinline__ uint8_t* bwd_smem(uint8_t* raw, int need, int smem_bytes,
                                             const DevCtl& ctl, int S) {
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
  if ((int)(smem - raw) + need > smem_bytes || S > kMaxTokens) {
    pdl_wait();
    if (threadIdx.x == 0) record_status(ctl, kStatusUnsupported);
    return nullptr;
  }
  return smem;
}

// ---------------------------------------------------------------- score pass

// The score pass's visited 128-key tiles of a row tile, in order (two per
// 256-key group).
__device__ __forceinline__ int next_tile128(const Ctl& c, uint32_t csq1, bool all_e, int kt,
                                            int S, int n_kt) {
  int t = kt + 1;
  while (t < n_kt) {
    if ((t & 1) != 0) return t;                 // the second tile of a visited group
    if (group_visible(c, csq1, all_e, t >> 1, S)) return t;
    t += 2;
  }
  return -1;
}

// Position in a cluster's run of the (batch, row tile, visited 128-key tile)
// sequence.  Every role walks the same run with its own copy.
struct TileWalk {
  int b, pair, kt, left;
  uint32_t csq1;
  bool all_e;
};

__device__ __forceinline__ void walk_enter(TileWalk& w, const Ctl& c, const int* pinfo,
                                           const uint16_t* codes, int j, int S, int n_kt,
                                           int tok_per_pair) {
  const int tq0 = w.pair * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
  w.csq1 = codes[tq1] >> 2;
  w.all_e = ((pinfo[w.pair] >> 30) & 1) != 0;
  w.kt = -1;
  for (int i = 0; i <= j; ++i) w.kt = next_tile128(c, w.csq1, w.all_e, w.kt, S, n_kt);
}

// Moves to the next tile of the run; returns true if the row tile changed.
__device__ __forceinline__ bool walk_next(TileWalk& w, const Ctl& c, const int* pinfo,
                                          const uint16_t* codes, int S, int n_kt, int n_pairs,
                                          int tok_per_pair) {
  if (--w.left <= 0) return false;
  const int nk = next_tile128(c, w.csq1, w.all_e, w.kt, S, n_kt);
  if (nk >= 0) {
    w.kt = nk;
    return false;
  }
  do {
    if (++w.pair == n_pairs) {
      w.pair = 0;
      ++w.b;
    }
  } while ((pinfo[w.pair] & 0x3FFFFFFF) == 0);
  walk_enter(w, c, pinfo, codes, 0, S, n_kt, tok_per_pair);
  return true;
}

// Score pass, at a row tile (b, pair): this row warp's share of its Q (parts
// 0, 1) or dO (parts 2, 3), a 256-byte slice of each of the warp's 32 rows,
// into TMEM lane quarter * 32 + row, 64 columns of bf16 pairs (the MMA's A
// layout).  Coalesced loads (8 rows x 64 B per instruction) become one row
// per lane through the warp's 2 KB stage (16-byte chunk j of row r at
// j ^ ((r / 2) % 4)); then the warp arrives on the leader's qd_full and warms
// L2 with the following row tile's rows (its Q / dO, lse, D).  Called only at
// row-tile switches, so it is kept out of line.
__device__ __noinline__ void score_copy_rows(const BwdTcParams& p, int b, int pair, uint32_t rank,
                                             int quarter, int part, uint32_t tmem,
                                             uint8_t* wstage, bool store_pending,
                                             const int* pinfo, int n_pairs, uint32_t qd_full_l) {
  const int lane = threadIdx.x & 31;
  const int rows_per_b = p.S * p.Hq;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const int r0 = pair * 2 * kRows + (int)rank * kRows + quarter * 32;
  const long long g0 = (long long)b * rows_per_b + r0;
  const uint8_t* gsrc = static_cast<const uint8_t*>(part < 2 ? p.q : p.dout) +
                        g0 * (long long)(kD * 2) + 256 * (part & 1);
  const uint32_t tdst = tmem + lane_off + 256 + 128 * (part >> 1) + 64 * (part & 1);
  if (store_pending) {   // the last P / dS box has been read out of the stage
    if (lane == 0) tma_store_wait_read();
    __syncwarp();
  }
#pragma unroll 1
  for (int h2 = 0; h2 < 2; ++h2) {
    uint4 qv[2][4];
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rr = 8 * i + (lane >> 2);
        qv[c2][i] = r0 + rr < rows_per_b
                        ? *reinterpret_cast<const uint4*>(gsrc + rr * (kD * 2) + 128 * h2 +
                                                          64 * c2 + 16 * (lane & 3))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rr = 8 * i + (lane >> 2);
        *reinterpret_cast<uint4*>(wstage + rr * 64 + (((lane & 3) ^ ((rr >> 1) & 3)) << 4)) =
            qv[c2][i];
      }
      __syncwarp();
      uint32_t r16[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 t4 =
            *reinterpret_cast<const uint4*>(wstage + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4));
        r16[4 * j] = t4.x; r16[4 * j + 1] = t4.y;
        r16[4 * j + 2] = t4.z; r16[4 * j + 3] = t4.w;
      }
      __syncwarp();
      tmem_st16(tdst + 32 * h2 + 16 * c2, r16);
    }
  }
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_remote(qd_full_l);
  if (p.mask_bs == 0 && (part & 1) == 0) {
    int nb = b, npair = pair;
    do {
      if (++npair == n_pairs) {
        npair = 0;
        ++nb;
      }
    } while (nb < p.B && (pinfo[npair] & 0x3FFFFFFF) == 0);
    const int nr0 = npair * 2 * kRows + (int)rank * kRows + quarter * 32;
    const int nrows = min(32, rows_per_b - nr0);
    if (nb < p.B && nrows > 0) {
      const long long ng0 = (long long)nb * rows_per_b + nr0;
      if (lane == 0)
        bulk_prefetch_l2(static_cast<const uint8_t*>(part < 2 ? p.q : p.dout) + ng0 * (kD * 2),
                         (uint32_t)nrows * (kD * 2));
      if (lane < nrows) prefetch_l2(part < 2 ? p.lse + ng0 + lane : p.D + ng0 + lane);
    }
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT1, 1)
    bwd_score_kernel(const __grid_constant__ BwdTcParams p, const DevCtl ctl, int smem_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int S = p.S, Hq = p.Hq;
  const int rows_per_b = S * Hq;
  const int n_pairs = (rows_per_b + 2 * kRows - 1) / (2 * kRows);
  uint8_t* smem = bwd_smem(smem_raw, smem_need(kOps1, S, n_pairs * 4), smem_bytes, ctl, S);
  if (smem == nullptr) return;
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kOps1);
  int* pinfo = reinterpret_cast<int*>(smem + kOps1 + ctl_bytes());
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOps1 + ctl_bytes() + pad128(n_pairs * 4));
  uint8_t* ring = smem;
  uint8_t* stage = ring + kNS1 * kStage1;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int tok_per_pair = 2 * kRows / Hq;
  const int n_sup = (S + kSup - 1) / kSup;
  const int n_kt = (S + kKT1 - 1) / kKT1;
  // A batch-shared mask: the clusters split the whole run evenly.  Per-batch
  // masks: one cluster per (batch, row tile), scanning its own batch row.
  const bool per_batch = p.mask_bs != 0;
  const int b_mask = per_batch ? cluster / n_pairs : 0;

  const uint8_t* ar_b = p.ar + (long long)b_mask * p.mask_bs;
  const int32_t* seg_b = p.seg ? p.seg + (long long)b_mask * p.mask_bs : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS1; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.qd_full, 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.s_free[i], 32);
    }
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_k64);
    tma_prefetch_desc(&p.map_v64);
    tma_prefetch_desc(&p.map_pw);
    tma_prefetch_desc(&p.map_dsw);
  }
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(&c.tmem_base, 512);
    tmem_relinquish_pair();
  }
  // Up to the wait below this kernel may overlap the previous one.  It reads
  // only ar_mask and the segment ids there, which no kernel of this library
  // writes; and it starts only after the backward's first launch (the
  // row-dot, which waits before it releases its dependents) has seen the
  // caller's earlier work complete.
  const Flags32 flags0 = load_flags32(ar_b, seg_b, S, (int)threadIdx.x * 32);
  build_codes_x32<kT1>(ar_b, seg_b, S, pad128(S), codes, c.scan, flags0,
                      TileSums{c.cs_first, c.cs_last, c.flags});
  // Per row tile: its visited key-tile count, and bit 30 if all its tokens
  // are experts (or padding).
  for (int pr = threadIdx.x; pr < n_pairs; pr += kT1) {
    const int tq0 = pr * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
    const bool all_e = tokens_all_expert_serial(codes, tq0, tq1);
    const uint32_t csq1 = codes[tq1] >> 2;
    int cnt = 0;
    for (int ks = 0; ks < n_sup; ++ks)
      if (group_visible(c, csq1, all_e, ks, S)) cnt += min(2 * ks + 2, n_kt) - 2 * ks;
    pinfo[pr] = cnt | (all_e ? (1 << 30) : 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();                 // the previous kernel's results are visible from here on
  pdl_launch_dependents();
  const uint32_t tmem = c.tmem_base;

  // This cluster's run.
  TileWalk w0{};
  {
    if (per_batch) {
      w0.b = b_mask;
      w0.pair = cluster % n_pairs;
      w0.left = pinfo[w0.pair] & 0x3FFFFFFF;
      if (w0.left > 0) walk_enter(w0, c, pinfo, codes, 0, S, n_kt, tok_per_pair);
    } else {
      long long Tb = 0;
      for (int pr = 0; pr < n_pairs; ++pr) Tb += pinfo[pr] & 0x3FFFFFFF;
      const long long T = Tb * p.B;
      const long long lo = T * cluster / n_clusters, hi = T * (cluster + 1) / n_clusters;
      w0.left = (int)(hi - lo);
      if (w0.left > 0) {
        w0.b = (int)(lo / Tb);
        long long r = lo - (long long)w0.b * Tb;
        w0.pair = 0;
        while (r >= (pinfo[w0.pair] & 0x3FFFFFFF)) {
          r -= pinfo[w0.pair] & 0x3FFFFFFF;
          ++w0.pair;
        }
        walk_enter(w0, c, pinfo, codes, (int)r, S, n_kt, tok_per_pair);
      }
    }
  }

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    // (Q and dO of each row tile reach TMEM through the row warps.)
    TileWalk w = w0;
    uint32_t n = 0;
    bool ok = true;
    // K and V are read by every row tile: keep them in L2 against the P and dS
    // stream this pass writes.
    const uint64_t keep = l2_policy_evict_last();
    while (w.left > 0 && ok) {
      const int s = (int)(n % kNS1);
      const uint32_t rel = n / kNS1;
      if (rel > 0 && !warp_wait(&c.empty[s], (rel - 1) & 1, c, ctl)) break;
      if (lane == 0) {
        const uint32_t full_l = mapa_shared(smem_u32(&c.full[s]), 0);
        if (leader) mbar_arrive_expect_tx(&c.full[s], 2 * kStage1);
        uint8_t* st = ring + s * kStage1;
        // this CTA's 64 keys of the tile, all 256 columns, of K and of V
        const int key0 = w.kt * kKT1 + 64 * (int)rank;
        tma_load_4d_pair_hint(st, &p.map_k64, full_l, 0, key0, 0, w.b, keep);
        tma_load_4d_pair_hint(st + kItem64, &p.map_v64, full_l, 0, key0, 0, w.b, keep);
      }
      __syncwarp();
      ++n;
      (void)walk_next(w, c, pinfo, codes, S, n_kt, n_pairs, tok_per_pair);
    }
    // Loads complete on the leader's barriers: wait there (bounded) for the
    // last phase of each, so no copy is in flight when the cluster leaves.
    if (leader && lane == 0) {
      for (int s = 0; s < kNS1; ++s) {
        const uint32_t n_s = n > (uint32_t)s ? (n - (uint32_t)s + kNS1 - 1) / kNS1 : 0;
        if (n_s > 0) (void)mbar_wait(&c.full[s], (n_s - 1) & 1, ctl);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- MMA issue (leader CTA only)
    if (leader) {
      const uint64_t rdesc = sdesc_sw128(smem_u32(ring), 16, 1024);
      const uint32_t tS = tmem, tP = tmem + 128, tQ = tmem + 256, tdO = tmem + 384;
      TileWalk w = w0;
      uint32_t n = 0, np = 0;
      bool new_pair = true, ok = true;
      while (w.left > 0 && ok) {
        // A new row tile: the row warps have put its Q and dO in TMEM.
        if (new_pair) {
          if (!warp_wait(&c.qd_full, np & 1, c, ctl)) break;
          ++np;
        }
        const int s = (int)(n % kNS1);
        if (!warp_wait(&c.full[s], (n / kNS1) & 1, c, ctl)) break;
        // S and dP have a TMEM buffer each, freed separately: the S MMAs of
        // tile n start once S of tile n - 1 has been read, while the row warps
        // still read dP (and the dP MMAs follow once they have), so the
        // tensor pipe need not idle while the row warps drain the tile.
        if (n >= 1 && !warp_wait(&c.s_free[0], (n - 1) & 1, c, ctl)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t kd = rdesc + (uint64_t)((s * kStage1) >> 4);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            // A: [128 rows x 16 d] of Q / dO in TMEM (a row per lane, bf16
            // pairs per column: a K step is 8 columns); B: [64 keys x 16 d] of
            // K / V, K-major, 8-row groups 1024 B apart, a K step walks 32 B
            // inside a 64-column block (8 KB), then to the next block.
            const uint32_t boff = (uint32_t)((kk >> 2) * (64 * 128) + (kk & 3) * 32);
            umma_pair_ts(tS, tQ + 8 * kk, kd + (boff >> 4), kIdescScore, kk > 0 ? 1u : 0u);
          }
          commit_both(&c.s_full[0]);
        }
        __syncwarp();
        if (n >= 1 && !warp_wait(&c.s_free[1], (n - 1) & 1, c, ctl)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t vd = rdesc + (uint64_t)((s * kStage1 + kItem64) >> 4);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t boff = (uint32_t)((kk >> 2) * (64 * 128) + (kk & 3) * 32);
            umma_pair_ts(tP, tdO + 8 * kk, vd + (boff >> 4), kIdescScore, kk > 0 ? 1u : 0u);
          }
          commit_both(&c.empty[s]);
          commit_both(&c.s_full[1]);
        }
        __syncwarp();
        ++n;
        new_pair = walk_next(w, c, pinfo, codes, S, n_kt, n_pairs, tok_per_pair);
      }
      if (lane == 0) umma_commit_pair(smem_u32(&c.drain));
      __syncwarp();
      (void)mbar_wait(&c.drain, 0, ctl);
    }
  } else {
    // ------------------------------------------ row warps (both CTAs)
    // A warp reaches only the TMEM lanes of quarter warp % 4; four warps share
    // each quarter's 32 rows, warp 2 + q + 4 h taking keys [32 h, 32 h + 32)
    // of every tile.  P = exp2(S c - lse) needs no running maximum, so the
    // warps never exchange anything.
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float cs = p.scale_log2;
    const uint32_t sS_free_l = mapa_shared(smem_u32(&c.s_free[0]), 0);
    const uint32_t dP_free_l = mapa_shared(smem_u32(&c.s_free[1]), 0);
    const uint32_t qd_full_l = mapa_shared(smem_u32(&c.qd_full), 0);
    // The warp's 32 x 32 P and dS boxes leave by TMA bulk stores from a 2 KB
    // stage laid out as the tensor map's 64-byte swizzle expects; the same
    // stage turns the row tile's Q / dO slabs into rows on their way to TMEM.
    uint8_t* wstage = stage + (warp - 2) * kBox1;
    const uint64_t stream = l2_policy_evict_first();
    bool store_pending = false;   // lane 0's bulk stores may still read the stage
    bool ok = true;

    TileWalk w = w0;
    uint32_t n = 0;
    // Per row tile: this thread's row.  Its lse and D are loaded when the row
    // tile is entered (right after its Q and dO copy) and first used after the
    // next S wait, which hides their latency.
    uint32_t csq = 0;
    bool row_expert = false, row_live = false;
    float lse = 0.f, Dv = 0.f;
    int rho0 = 0;                                           // the warp's row 0 in its batch element
    auto enter_row_tile = [&](const TileWalk& t) {
      score_copy_rows(p, t.b, t.pair, rank, quarter, part, tmem, wstage, store_pending, pinfo,
                      n_pairs, qd_full_l);
      store_pending = false;   // the copy waited for the stage
      rho0 = t.pair * 2 * kRows + (int)rank * kRows + quarter * 32;
      const int rho = rho0 + lane;
      const bool row_valid = rho < rows_per_b;
      const int tq1 = min(t.pair * tok_per_pair + tok_per_pair, S) - 1;
      const uint32_t cq = codes[row_valid ? rho / Hq : tq1];
      csq = cq >> 2;
      row_expert = (cq & 2u) != 0;
      row_live = row_valid && !is_pad(cq);
      const long long g0 = (long long)t.b * rows_per_b + rho0;
      lse = row_live ? p.lse[g0 + lane] : 0.f;
      Dv = row_live ? p.D[g0 + lane] : 0.f;
    };
    if (w.left > 0) enter_row_tile(w);
    while (w.left > 0 && ok) {
      const int k0 = w.kt * kKT1;
      const int kh = k0 + 32 * part;                        // this warp's first key
      // Keys of this tile the row sees: a prefix (block index is
      // non-decreasing), minus FAST keys for expert rows and padding keys.
      // The tile's last key visible means every key is (most tiles).
      int e = kKT1;
      if ((uint32_t)(codes[min(k0 + kKT1, S) - 1] >> 2) > csq) {
        e = 0;
#pragma unroll
        for (int step = kKT1; step >= 1; step >>= 1) {
          const int probe = e + step;
          if (probe <= kKT1 && (uint32_t)(codes[k0 + probe - 1] >> 2) <= csq) e = probe;
        }
      }
      e = row_live ? min(e, S - k0) - 32 * part : 0;       // visible keys of this warp's 32
      const uint32_t tf = c.flags[w.kt];
      const bool hole = ((tf & 1u) && row_expert) || (tf & 4u);
      if (!warp_wait(&c.s_full[0], n & 1, c, ctl)) break;
      tc_fence_after();
      const float lse2 = lse * kLog2e;
      // S first: P is formed while the dP MMAs run.
      uint32_t s0[32];
      tmem_ld32(tmem + lane_off + 32 * part, s0);
      tmem_ld_wait();
      reg_fence(s0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(sS_free_l);
      uint32_t hid = 0u;               // bit j: key kh + j hidden by the hole rule
      if (hole) {
        const uint4* kc = reinterpret_cast<const uint4*>(codes + kh);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const uint4 v4 = kc[q8];
          const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const uint32_t ck = (wv[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
            const uint32_t hide = ((row_expert && (ck & 1u)) || is_pad(ck)) ? 1u : 0u;
            hid |= hide << (8 * q8 + h);
          }
        }
      }
      // P in place of S (fp32; exact zeros where the key is hidden).
      uint32_t pk[16], dk[16];
      if (__all_sync(0xffffffffu, e >= 32 && hid == 0u)) {
        // Every row of the warp sees all 32 keys (most tiles): no predicates.
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 t = ffma2(make_float2(__uint_as_float(s0[j]), __uint_as_float(s0[j + 1])),
                                 make_float2(cs, cs), make_float2(-lse2, -lse2));
          s0[j] = __float_as_uint(ex2(t.x));
          s0[j + 1] = __float_as_uint(ex2(t.y));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 t = ffma2(make_float2(__uint_as_float(s0[j]), __uint_as_float(s0[j + 1])),
                                 make_float2(cs, cs), make_float2(-lse2, -lse2));
          s0[j] = __float_as_uint((j < e && !((hid >> j) & 1u)) ? ex2(t.x) : 0.f);
          s0[j + 1] = __float_as_uint((j + 1 < e && !((hid >> (j + 1)) & 1u)) ? ex2(t.y) : 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        pk[j >> 1] = cvt_bf16x2(__uint_as_float(s0[j]), __uint_as_float(s0[j + 1]));
      // Row `lane` of each 32 x 32 box: its 16-byte chunk j at j ^ ((lane / 2) % 4).
      // Rows past the batch element's end are clipped by the tensor map.
      const bool do_store = rho0 < rows_per_b && kh < p.Skp;
      auto store_box = [&](const uint32_t* src, const CUtensorMap* map) {
        uint8_t* const line = wstage + lane * 64;
        if (store_pending) {   // the previous box has been read out of the stage
          if (lane == 0) tma_store_wait_read();
          __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(line + ((j ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(src[4 * j], src[4 * j + 1], src[4 * j + 2], src[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d_hint(map, wstage, kh, rho0, w.b, stream);
          tma_store_commit();
        }
        __syncwarp();
        store_pending = true;
      };
      if (do_store) store_box(pk, &p.map_pw);
      if (!warp_wait(&c.s_full[1], n & 1, c, ctl)) break;
      tc_fence_after();
      uint32_t d0[32];
      tmem_ld32(tmem + lane_off + 128 + 32 * part, d0);
      tmem_ld_wait();
      reg_fence(d0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(dP_free_l);
      {
        const float2 nD = make_float2(-Dv, -Dv);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 dd = fadd2(make_float2(__uint_as_float(d0[j]), __uint_as_float(d0[j + 1])),
                                  nD);
          dk[j >> 1] = cvt_bf16x2(__uint_as_float(s0[j]) * dd.x,
                                  __uint_as_float(s0[j + 1]) * dd.y);
        }
      }
      if (do_store) store_box(dk, &p.map_dsw);
      // The next tile; when it starts a new row tile, its Q and dO go to TMEM
      // now (every MMA that read the old ones has completed: dP is here).
      TileWalk nw = w;
      const bool next_new = walk_next(nw, c, pinfo, codes, S, n_kt, n_pairs, tok_per_pair);
      if (next_new) enter_row_tile(nw);
      ++n;
      w = nw;
    }
    if (store_pending && lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------------- dK/dV pass

// Warp-collective: 1 if every token of [tq0, tq1] is an expert (or padding)
// token.
__device__ __forceinline__ bool tokens_all_expert(const uint16_t* codes, int tq0, int tq1,
                                                  int lane) {
  int all_e = 1;
  for (int t = tq0 + lane; t <= tq1; t += 32) all_e &= (codes[t] >> 1) & 1;
  return __all_sync(0xffffffffu, all_e) != 0;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ BwdTcParams p, const DevCtl ctl, int smem_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = bwd_smem(smem_raw, smem_need(kOps2, p.S, 0), smem_bytes, ctl, p.S);
  if (smem == nullptr) return;
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kOps2);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOps2 + ctl_bytes());
  uint8_t* ring = smem;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, Hq = p.Hq;
  const int rows_per_b = S * Hq;
  const int n_pairs = (rows_per_b + 2 * kRows - 1) / (2 * kRows);
  const int n_sup = (S + kSup - 1) / kSup;
  const int unit = blockIdx.x >> 1;
  const int chunk = unit % p.n_chunks;
  const int ks = (unit / p.n_chunks) % n_sup;
  const int b = unit / p.n_chunks / n_sup;
  const int p_begin = chunk * p.pairs_per_chunk;
  const int p_end = min(p_begin + p.pairs_per_chunk, n_pairs);
  const int tok_per_pair = 2 * kRows / Hq;

  const uint8_t* ar_b = p.ar + (long long)b * p.mask_bs;
  const int32_t* seg_b = p.seg ? p.seg + (long long)b * p.mask_bs : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS2; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.done[0], 1);
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_pT);
    tma_prefetch_desc(&p.map_dsT);
    tma_prefetch_desc(&p.map_qh);
    tma_prefetch_desc(&p.map_doh);
  }
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(&c.tmem_base, 512);
    tmem_relinquish_pair();
  }
  // Up to the wait below this kernel may overlap the previous one.  It reads
  // only ar_mask and the segment ids there, which no kernel of this library
  // writes; and it starts only after the backward's first launch (the
  // row-dot, which waits before it releases its dependents) has seen the
  // caller's earlier work complete.
  const Flags32 flags0 = load_flags32(ar_b, seg_b, S, (int)threadIdx.x * 32);
  build_codes_x32<kT>(ar_b, seg_b, S, pad128(S), codes, c.scan, flags0,
                      TileSums{c.cs_first, c.cs_last, c.flags});
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();                 // the previous kernel's results are visible from here on
  pdl_launch_dependents();
  const uint32_t tmem = c.tmem_base;
  const uint32_t tdV = tmem, tdK = tmem + 256;

  // The 64-row steps of this unit: every step of each row tile in
  // [p_begin, p_end) that may see a key of group ks (the same rule the score
  // pass used to decide which groups it wrote).
  auto tile_steps = [&](int pt) -> int {
    const int tq0 = pt * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
    const bool all_e = tokens_all_expert(codes, tq0, tq1, lane);
    if (!group_visible(c, (uint32_t)(codes[tq1] >> 2), all_e, ks, S)) return 0;
    return (min(2 * kRows, rows_per_b - pt * 2 * kRows) + 63) / 64;
  };

  uint32_t n_total = 0;     // steps this unit runs (each role counts them)
  if (warp == 0) {
    // ---------------------------------------------------------- producer
    bool ok = true;
    for (int pt = p_begin; pt < p_end && ok; ++pt) {
      const int nst = tile_steps(pt);
      for (int st = 0; st < nst && ok; ++st, ++n_total) {
        const uint32_t n = n_total;
        const int s = (int)(n % kNS2);
        const uint32_t rel = n / kNS2;
        if (rel > 0 && !warp_wait(&c.empty[s], (rel - 1) & 1, c, ctl)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t full_l = mapa_shared(smem_u32(&c.full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&c.full[s], 2 * kStage2);
          uint8_t* sg = ring + s * kStage2;
          const int r0 = pt * 2 * kRows + 64 * st;
          const int kb = 4 * ks + 2 * (int)rank;       // this CTA's 128 keys: 2 blocks of 64
          tma_load_4d_pair(sg, &p.map_pT, full_l, 0, r0, kb, b);
          tma_load_4d_pair(sg + kHalf64, &p.map_dsT, full_l, 0, r0, kb, b);
          tma_load_4d_pair(sg + 2 * kHalf64, &p.map_doh, full_l, 0, r0, 2 * (int)rank, b);
          tma_load_4d_pair(sg + 3 * kHalf64, &p.map_qh, full_l, 0, r0, 2 * (int)rank, b);
        }
        __syncwarp();
      }
    }
    if (leader && lane == 0) {
      for (int s = 0; s < kNS2; ++s) {
        const uint32_t n_s = n_total > (uint32_t)s ? (n_total - (uint32_t)s + kNS2 - 1) / kNS2 : 0;
        if (n_s > 0) (void)mbar_wait(&c.full[s], (n_s - 1) & 1, ctl);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- MMA issue (leader CTA only)
    for (int pt = p_begin; pt < p_end; ++pt) n_total += (uint32_t)tile_steps(pt);
    if (leader) {
      const uint64_t rdesc = sdesc_sw128(smem_u32(ring), kHalf64 / 2, 1024);
      uint32_t n = 0;
      bool ok = true;
      for (; n < n_total && ok; ++n) {
        const int s = (int)(n % kNS2);
        if (!warp_wait(&c.full[s], (n / kNS2) & 1, c, ctl)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t base = (uint32_t)(s * kStage2);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            // A = P^T / dS^T [128 keys x 16 rows] per CTA, B = dO / Q [16 rows x
            // (128 columns per CTA)], both MN-major: 8-row groups 1024 B apart,
            // 64-wide blocks 8 KB apart; a K step is 16 rows (2048 B).
            const uint32_t ko = (uint32_t)(k4 * 2048);
            umma_pair_ss(tdV, rdesc + ((base + ko) >> 4),
                         rdesc + ((base + 2 * kHalf64 + ko) >> 4), kIdescKV,
                         (n > 0 || k4 > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t ko = (uint32_t)(k4 * 2048);
            umma_pair_ss(tdK, rdesc + ((base + kHalf64 + ko) >> 4),
                         rdesc + ((base + 3 * kHalf64 + ko) >> 4), kIdescKV,
                         (n > 0 || k4 > 0) ? 1u : 0u);
          }
          commit_both(&c.empty[s]);
          if (n + 1 == n_total) commit_both(&c.done[0]);
        }
        __syncwarp();
      }
      if (lane == 0) umma_commit_pair(smem_u32(&c.drain));
      __syncwarp();
      (void)mbar_wait(&c.drain, 0, ctl);
    }
  } else {
    // ------------------------------------ epilogue warps (both CTAs)
    for (int pt = p_begin; pt < p_end; ++pt) n_total += (uint32_t)tile_steps(pt);
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int key0 = ks * kSup + (int)rank * kRows + quarter * 32;   // the warp's first key
    const bool have = n_total > 0;
    bool ok = true;
    if (have) {
      ok = warp_wait(&c.done[0], 0, c, ctl);
      tc_fence_after();
    }
    if (ok) {
      // Every MMA has completed, so the ring is free: each warp transposes
      // its rows through its own 4 KB of it.
      uint8_t* wstage = ring + quarter * kWarpStage;
      float* dkbase;
      float* dvbase;
      uint32_t valid;
      if (p.n_chunks == 1) {
        valid = __ballot_sync(0xffffffffu, key0 + lane < S);
        const long long o = ((long long)b * S + key0) * kD;
        dkbase = p.dk + o;
        dvbase = p.dv + o;
      } else {
        valid = 0xffffffffu;
        const long long kpad = (long long)n_sup * kSup;
        const long long o = (((long long)chunk * p.B + b) * kpad + key0) * kD;
        dkbase = p.part + o;
        dvbase = p.part + (long long)p.n_chunks * p.B * kpad * kD + o;
      }
      tmem_rows_out(tdK + lane_off, p.scale, wstage, valid, lane, !have,
                    [&](int rr) { return dkbase + (long long)rr * kD; });
      tmem_rows_out(tdV + lane_off, 1.f, wstage, valid, lane, !have,
                    [&](int rr) { return dvbase + (long long)rr * kD; });
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ----------------------------------------------------------------- dQ pass

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT, 1)
    bwd_dq_tc_kernel(const __grid_constant__ BwdTcParams p, const DevCtl ctl, int smem_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = bwd_smem(smem_raw, smem_need(kOps3, p.S, 0), smem_bytes, ctl, p.S);
  if (smem == nullptr) return;
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kOps3);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOps3 + ctl_bytes());
  uint8_t* ring = smem;
  uint8_t* stage = smem + kNS3 * kStage3;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, Hq = p.Hq;
  const int rows_per_b = S * Hq;
  const int n_pairs = (rows_per_b + 2 * kRows - 1) / (2 * kRows);
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int n_units = p.B * n_pairs;
  const int tok_per_pair = 2 * kRows / Hq;
  const int n_kt = (S + kKT - 1) / kKT;
  // A batch-shared mask: clusters walk units c, c + C, ...; per-batch masks:
  // one unit per cluster, which scans that unit's batch row.
  const bool per_batch = p.mask_bs != 0;
  const int b_mask = per_batch ? cluster / n_pairs : 0;

  const uint8_t* ar_b = p.ar + (long long)b_mask * p.mask_bs;
  const int32_t* seg_b = p.seg ? p.seg + (long long)b_mask * p.mask_bs : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS3; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&c.done[a], 1);
      mbar_init(&c.acc_free[a], 8);
    }
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_ds);
    tma_prefetch_desc(&p.map_kh);
  }
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(&c.tmem_base, 512);
    tmem_relinquish_pair();
  }
  // Up to the wait below this kernel may overlap the previous one.  It reads
  // only ar_mask and the segment ids there, which no kernel of this library
  // writes; and it starts only after the backward's first launch (the
  // row-dot, which waits before it releases its dependents) has seen the
  // caller's earlier work complete.
  const Flags32 flags0 = load_flags32(ar_b, seg_b, S, (int)threadIdx.x * 32);
  build_codes_x32<kT>(ar_b, seg_b, S, pad128(S), codes, c.scan, flags0,
                      TileSums{c.cs_first, c.cs_last, c.flags});
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();                 // the previous kernel's results are visible from here on
  pdl_launch_dependents();
  const uint32_t tmem = c.tmem_base;

  // Visited key tiles of row tile `pair`: kt = first, then next_tile.
  auto pair_info = [&](int pair, uint32_t& csq1, bool& all_e) {
    const int tq0 = pair * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
    csq1 = codes[tq1] >> 2;
    all_e = tokens_all_expert(codes, tq0, tq1, lane);
  };
  const int u_first = cluster, u_step = per_batch ? n_units : n_clusters;

  if (warp == 0) {
    uint32_t n = 0;
    bool ok = true;
    for (int u = u_first; u < n_units && ok; u += u_step) {
      const int pair = u % n_pairs, b = u / n_pairs;
      const int row0 = pair * 2 * kRows + (int)rank * kRows;
      uint32_t csq1;
      bool all_e;
      pair_info(pair, csq1, all_e);
      for (int kt = next_tile(c, csq1, all_e, -1, S, n_kt); kt >= 0 && ok;
           kt = next_tile(c, csq1, all_e, kt, S, n_kt), ++n) {
        const int s = (int)(n % kNS3);
        const uint32_t rel = n / kNS3;
        if (rel > 0 && !warp_wait(&c.empty[s], (rel - 1) & 1, c, ctl)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t full_l = mapa_shared(smem_u32(&c.full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&c.full[s], 2 * kStage3);
          uint8_t* sg = ring + s * kStage3;
          tma_load_4d_pair(sg, &p.map_ds, full_l, 0, row0, kt, b);
          tma_load_4d_pair(sg + kDsTile, &p.map_kh, full_l, 0, kt * kKT, 2 * (int)rank, b);
        }
        __syncwarp();
      }
    }
    if (leader && lane == 0) {
      for (int s = 0; s < kNS3; ++s) {
        const uint32_t n_s = n > (uint32_t)s ? (n - (uint32_t)s + kNS3 - 1) / kNS3 : 0;
        if (n_s > 0) (void)mbar_wait(&c.full[s], (n_s - 1) & 1, ctl);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader) {
      const uint64_t adesc = sdesc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t bdesc = sdesc_sw128(smem_u32(ring), kHalf64 / 2, 1024);
      uint32_t n = 0, i = 0;
      bool ok = true;
      for (int u = u_first; u < n_units && ok; u += u_step, ++i) {
        const int a = (int)(i & 1);
        // Accumulator a was last read by the epilogue of unit i - 2.
        if (i >= 2 && !warp_wait(&c.acc_free[a], ((i - 2) >> 1) & 1, c, ctl)) break;
        const int pair = u % n_pairs;
        uint32_t csq1;
        bool all_e;
        pair_info(pair, csq1, all_e);
        uint32_t t = 0;
        for (int kt = next_tile(c, csq1, all_e, -1, S, n_kt); kt >= 0;
             kt = next_tile(c, csq1, all_e, kt, S, n_kt), ++n, ++t) {
          const int s = (int)(n % kNS3);
          if (!warp_wait(&c.full[s], (n / kNS3) & 1, c, ctl)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t base = (uint32_t)(s * kStage3);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              // A = dS [128 rows x 16 keys] K-major (a K step walks 32 B of
              // the 128-byte line); B = K [16 keys x (128 columns per CTA)]
              // MN-major.
              umma_pair_ss(tmem + 256 * a, adesc + ((base + k4 * 32) >> 4),
                           bdesc + ((base + kDsTile + k4 * 2048) >> 4), kIdescQ,
                           (t > 0 || k4 > 0) ? 1u : 0u);
            }
            commit_both(&c.empty[s]);
          }
          __syncwarp();
        }
        if (!ok) break;
        // A unit without tiles still completes a phase of done[a].
        if (lane == 0) commit_both(&c.done[a]);
        __syncwarp();
      }
      if (lane == 0) umma_commit_pair(smem_u32(&c.drain));
      __syncwarp();
      (void)mbar_wait(&c.drain, 0, ctl);
    }
  } else {
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t* wstage = stage + quarter * kWarpStage;
    const uint32_t acc_free_l0 = mapa_shared(smem_u32(&c.acc_free[0]), 0);
    const uint32_t acc_free_l1 = mapa_shared(smem_u32(&c.acc_free[1]), 0);
    uint32_t i = 0;
    for (int u = u_first; u < n_units; u += u_step, ++i) {
      const int a = (int)(i & 1);
      const int pair = u % n_pairs, b = u / n_pairs;
      uint32_t csq1;
      bool all_e;
      pair_info(pair, csq1, all_e);
      const bool have = next_tile(c, csq1, all_e, -1, S, n_kt) >= 0;
      if (!warp_wait(&c.done[a], (i >> 1) & 1, c, ctl)) break;
      tc_fence_after();
      const int rho0 = pair * 2 * kRows + (int)rank * kRows + quarter * 32;
      const uint32_t valid = __ballot_sync(0xffffffffu, rho0 + lane < rows_per_b);
      float* base = p.dq + ((long long)b * rows_per_b + rho0) * kD;
      tmem_rows_out(tmem + 256 * a + lane_off, p.scale, wstage, valid, lane, !have,
                    [&](int rr) { return base + (long long)rr * kD; });
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(a ? acc_free_l1 : acc_free_l0);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------- small kernels

// D[row] = sum_d dO[row, d] * O[row, d] in fp32: one warp per row, each lane
// 8 of the 256 columns (16-byte loads).
__global__ void __launch_bounds__(256)
    bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ out,
                      const __nv_bfloat16* __restrict__ dout, float* __restrict__ D,
                      long long n_rows) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < n_rows; row += warps) {
    const uint4 a = reinterpret_cast<const uint4*>(out + row * kD)[lane];
    const uint4 g = reinterpret_cast<const uint4*>(dout + row * kD)[lane];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[i]));
      s = fmaf(af.x, gf.x, s);
      s = fmaf(af.y, gf.y, s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) D[row] = s;
  }
}

// dk, dv = the sums over row chunks of the dK/dV pass's partials, added in
// chunk order (deterministic).
__global__ void __launch_bounds__(256)
    bwd_chunk_sum_kernel(const float* __restrict__ part, float* __restrict__ dk,
                         float* __restrict__ dv, int n_chunks, int B, int S, int kpad) {
  pdl_wait();                 // the partials come from the dK/dV pass before
  pdl_launch_dependents();
  const long long n4 = (long long)B * S * (kD / 4);
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long per_chunk = (long long)B * kpad * kD;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const long long c4 = i % (kD / 4);
    const long long bk = i / (kD / 4);            // b * S + key
    const long long b = bk / S, key = bk - b * S;
    const long long o = (b * kpad + key) * kD + 4 * c4;
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
    for (int ch = 0; ch < n_chunks; ++ch) {
      const float4 a = *reinterpret_cast<const float4*>(part + ch * per_chunk + o);
      const float4 v = *reinterpret_cast<const float4*>(part + (n_chunks + ch) * per_chunk + o);
      sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
      sv.x += v.x; sv.y += v.y; sv.z += v.z; sv.w += v.w;
    }
    reinterpret_cast<float4*>(dk)[i] = sk;
    reinterpret_cast<float4*>(dv)[i] = sv;
  }
}

template <typename K>
cudaError_t launch_cluster_kernel(K kernel, int clusters, int need, const BwdTcParams& p,
                                  const DevCtl& ctl, cudaStream_t st, int threads = kT) {
  static_assert(sizeof(BwdTcParams) <= 4096, "kernel parameters too large");
  const int smem = min(need + 1024, kSmemLimit);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemLimit);
  if (e != cudaSuccess) return e;
  return launch_pdl(kernel, dim3(2 * clusters), dim3(threads), smem, st, p, ctl, smem);
}

}  // namespace

BwdTcPlan bwd_tc_plan(int B, int S, int Hq, int sms) {
  BwdTcPlan pl{};
  const int rows = S * Hq;
  pl.n_pairs = (rows + 2 * kRows - 1) / (2 * kRows);
  pl.n_sup = (S + kSup - 1) / kSup;
  pl.Skp = (S + kKT - 1) / kKT * kKT;
  pl.clusters = max(sms / 2, 1);
  // Row chunks of the dK/dV pass: the fewest that keep the SM pairs as busy
  // as any larger count would (whole waves of clusters).
  const long long units = (long long)B * pl.n_sup;
  int best = 1;
  double best_t = 1e30;
  for (int c = 1; c <= pl.n_pairs && c <= 64; ++c) {
    const int ppc = (pl.n_pairs + c - 1) / c;
    const int cc = (pl.n_pairs + ppc - 1) / ppc;                  // chunks actually used
    const double waves = (double)((units * cc + pl.clusters - 1) / pl.clusters);
    const double t = waves * ppc;
    if (t < best_t - 1e-9) {
      best_t = t;
      best = cc;
    }
  }
  pl.pairs_per_chunk = (pl.n_pairs + best - 1) / best;
  pl.n_chunks = (pl.n_pairs + pl.pairs_per_chunk - 1) / pl.pairs_per_chunk;
  const size_t a = 256;
  auto up = [&](size_t x) { return (x + a - 1) / a * a; };
  pl.off_D = 0;
  pl.off_P = up((size_t)B * rows * sizeof(float));
  pl.off_dS = pl.off_P + up((size_t)B * rows * pl.Skp * 2);
  pl.off_part = pl.off_dS + up((size_t)B * rows * pl.Skp * 2);
  const size_t part = pl.n_chunks > 1
                          ? (size_t)2 * pl.n_chunks * B * pl.n_sup * kSup * kD * sizeof(float)
                          : 0;
  pl.bytes = pl.off_part + up(part);
  return pl;
}

cudaError_t launch_backward_tc(const BwdTcParams& p, const DevCtl& ctl, cudaStream_t st) {
  const long long rows = (long long)p.B * p.S * p.Hq;
  const int rd_blocks = (int)min((rows + 7) / 8, (long long)148 * 16);
  cudaError_t e = launch_pdl(bwd_rowdot_kernel, dim3(rd_blocks), dim3(256), 0, st,
                             static_cast<const __nv_bfloat16*>(p.out),
                             static_cast<const __nv_bfloat16*>(p.dout), const_cast<float*>(p.D),
                             rows);
  if (e != cudaSuccess) return e;
  const int n_pairs = (p.S * p.Hq + 2 * kRows - 1) / (2 * kRows);
  const int n_sup = (p.S + kSup - 1) / kSup;
  const int units = p.B * n_pairs;
  const int persistent = p.mask_bs == 0 ? min(units, p.clusters) : units;
  e = launch_cluster_kernel(bwd_score_kernel, persistent,
                            smem_need(kOps1, p.S, n_pairs * 4), p, ctl, st, kT1);
  if (e != cudaSuccess) return e;
  e = launch_cluster_kernel(bwd_dkdv_tc_kernel, p.B * n_sup * p.n_chunks,
                            smem_need(kOps2, p.S, 0), p, ctl, st);
  if (e != cudaSuccess) return e;
  if (p.n_chunks > 1) {
    const long long n4 = (long long)p.B * p.S * (kD / 4);
    const int blocks = (int)min((n4 + 255) / 256, (long long)148 * 8);
    e = launch_pdl(bwd_chunk_sum_kernel, dim3(blocks), dim3(256), 0, st,
                   static_cast<const float*>(p.part), p.dk, p.dv, p.n_chunks, p.B, p.S,
                   n_sup * kSup);
    if (e != cudaSuccess) return e;
  }
  return launch_cluster_kernel(bwd_dq_tc_kernel, persistent, smem_need(kOps3, p.S, 0), p, ctl,
                               st);
}

}  // namespace piattn
