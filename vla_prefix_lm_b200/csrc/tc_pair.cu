// tc_pair.cu -- bf16 joint (prefix-LM) attention on tcgen05, CTA-pair (2-SM) form.
//
// A cluster of two CTAs computes 256-row query tiles: 256 / Hq query tokens x
// Hq heads, 128 rows per CTA.  With a single KV head all rows read the same
// K/V rows ("π0.5 vs MM-DiT joint attention", "joint attention 只管算子": 8
// query heads, 1 KV head, head_dim 256, one shared KV pool).
//
// Per key tile of 128 keys, issued for the pair by two threads of the even CTA
// (one for QK, one for PV):
//   S = Q K^T   tcgen05.mma.cta_group::2, M = 256: A = Q rows of each CTA
//               (its shared memory), B = K split by keys (64 per CTA)
//   P           fp32 online softmax in each CTA, one thread per row; P is
//               written to shared memory as bf16 and S's TMEM is released as
//               soon as it has been read, so QK of the next tiles never waits
//               for a PV
//   O += P V    tcgen05.mma.cta_group::2: A = P (each CTA's shared memory),
//               B = V split by columns (128 of the 256 per CTA)
// Each SM streams half of every K/V tile, and every MMA instruction and every
// barrier round trip covers twice the work of a one-CTA, 64-key design.
//
// Work units.  A unit is one (batch, 256-row query tile, key split).  When
// ar_mask / segment_ids are shared by the batch, one cluster per SM pair runs
// and walks units c, c + C, c + 2C, ...: the next unit's Q is loaded as soon
// as the last QK of the current one has read Q, its first QKs run while the
// softmax warps write the current unit's output, and the mask scan runs once
// per cluster.  With per-batch masks every unit gets its own cluster.
//
// Mask: every CTA scans ar_mask / segment_ids into packed per-token codes
// (mask.cuh).  Per unit, each warp classifies every key tile for the unit's
// 256 query rows (skip / full / partial) into its own list -- all lists are
// equal, and private lists need no cross-warp synchronisation -- and a
// partial tile is masked per row by its visible-prefix length plus, for
// expert rows, the FAST keys.  No mask is materialised.
//
// Warp roles per CTA (224 threads):
//   warp 0      TMA producer for this CTA's halves (both CTAs)
//   warp 1      TMEM allocation (both CTAs, cta_group::2); QK issue (even CTA)
//   warps 2..5  softmax, O correction, epilogue (both CTAs, own rows)
//   warp 6      PV issue (even CTA)
//
// TMEM per CTA (512 columns): O fp32 [0,256) | S0 [256,384) | S1 [384,512).
// Shared memory per CTA: Q 64 KB | K ring 2 x 32 KB (this CTA's 64 keys x
// 256) | V ring 2 or 4 x 16 KB (64 keys x this CTA's 128 columns) | P 32 KB
// ([128 rows x 128 keys] bf16, two 128-byte-swizzled [128 x 64] blocks; also
// the output staging area) | control | per-token codes.
//
// Synchronisation across the pair: the even CTA owns q_full, k_full, v_full,
// s_free, p_full and o_free (the odd CTA's TMA loads and softmax warps arrive
// there through cluster addresses); the issuing threads' commits arrive on
// the q_empty, k_empty, v_empty, s_full and o_done barriers of both CTAs.
// Every wait is bounded (DevCtl).  Counters that index barriers and ring
// slots run across units; each ring has a single consumer thread, which
// waits on its slots in fill order.
#include <atomic>
#include <cfloat>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kThreads = 224;
constexpr int kBM = 128;                    // query rows per CTA (256 per pair)
constexpr int kBN = 128;                    // keys per key tile
constexpr int kD = 256;
constexpr int kQBlk = kBM * 128;            // [128 rows x 64 bf16] = 16 KB
constexpr int kQBytes = 4 * kQBlk;          // 64 KB
constexpr int kKBlk = 64 * 128;             // K item block: [64 keys x 64 d] = 8 KB
constexpr int kKItem = 4 * kKBlk;           // K item: this CTA's 64 keys x 256 d = 32 KB
constexpr int kVBlk = 64 * 128;             // V item block: [64 keys x 64 d] = 8 KB
constexpr int kVItem = 2 * kVBlk;           // V item: 64 keys x this CTA's 128 d = 16 KB
constexpr int kPBlk = kBM * 128;            // P block: [128 rows x 64 keys] = 16 KB
constexpr int kPBytes = 2 * kPBlk;          // 32 KB
constexpr int kStageRows = 32;              // output rows staged per softmax warp
constexpr int kOffQ = 0;
constexpr int kOffRing = kQBytes;
constexpr int kLists = 6;                   // tile lists of warps 0 and 2..5
constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays <= 256
constexpr int kSmemLimit = 232448;          // 227 KB per CTA on sm_100

constexpr uint32_t kIdescQK = idesc_bf16_f32(2 * kBM, kBN, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(2 * kBM, kD, false, true);
constexpr uint32_t kColO = 0, kColS = 256;

constexpr uint16_t kTilePartial = 0x8000;
constexpr uint16_t kTileAnyFast = 0x4000;
constexpr uint16_t kTileAnyPad = 0x2000;
constexpr uint16_t kTileIndex = 0x1FFF;

// Shared-memory layout: a ring of kK K items (32 KB) and a ring of kV V
// items (16 KB, half a key tile each), and up to kMaxTok tokens of per-token
// codes.  Each ring has one consumer thread.  Four V slots (two key tiles)
// fit beside Q and P only for short sequences.
template <int kK_, int kV_, int kMaxTok_>
struct Layout {
  static constexpr int kK = kK_;
  static constexpr int kV = kV_;
  static constexpr int kMaxTok = kMaxTok_;
  static constexpr int kMaxKeyTiles = (kMaxTok + kBN - 1) / kBN + 2;
  static constexpr int kOffV = kOffRing + kK * kKItem;
  static constexpr int kOffP = kOffV + kV * kVItem;
  static constexpr int kOffCtl = kOffP + kPBytes;
};

template <class L>
struct __align__(8) Smem {
  static constexpr int kMaxKeyTiles = L::kMaxKeyTiles;
  uint64_t q_full;               // even CTA: both Q halves landed (one phase per unit)
  uint64_t q_empty;              // each CTA: the unit's last QK has read Q
  uint64_t k_full[L::kK];        // even CTA: both CTAs' K items landed
  uint64_t k_empty[L::kK];       // each CTA: its K slot may be refilled
  uint64_t v_full[L::kV];        // even CTA: both CTAs' V items landed
  uint64_t v_empty[L::kV];       // each CTA: its V slot may be refilled
  uint64_t s_full[2];            // each CTA: S tile in its TMEM
  uint64_t s_free[2];            // even CTA: the pair's 8 softmax warps have read S
  uint64_t p_full;               // even CTA: P written by the pair's 8 softmax warps
  uint64_t o_done;               // each CTA: PV finished
  uint64_t o_free;               // even CTA: the pair's softmax warps have read O
  uint64_t drain_qk;             // even CTA: every QK issued has completed
  uint64_t drain_pv;             // even CTA: every PV issued has completed
  uint32_t tmem_base;
  int abort;
  int scan[kThreads / 32];
  uint16_t list[kLists][kMaxKeyTiles];
  uint16_t tile_cs_first[kMaxKeyTiles];
  uint16_t tile_cs_last[kMaxKeyTiles];
  uint8_t tile_fast[kMaxKeyTiles];
};

template <class L>
__host__ __device__ constexpr int off_codes() {
  return L::kOffCtl + ((int)sizeof(Smem<L>) + 127) / 128 * 128;
}

__host__ __device__ constexpr int pad_tokens(int n) { return (n + 127) / 128 * 128; }

// Bytes a layout needs past a 1024-byte aligned base.
template <class L>
__host__ __device__ constexpr int layout_bytes(int n_code_tokens) {
  return off_codes<L>() + pad_tokens(n_code_tokens) * 2;
}

using LayoutLong = Layout<2, 2, kMaxTokens>;   // any length
using LayoutShort = Layout<2, 4, 768>;         // short sequences (<= 768 tokens)
static_assert(layout_bytes<LayoutLong>(kMaxTokens) <= kSmemLimit, "layout too large");
static_assert(layout_bytes<LayoutShort>(768) + 1024 <= kSmemLimit, "short layout too large");

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

// Warp-uniform bounded wait: every lane polls, all lanes get the same answer.
template <class SmemT>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, SmemT& sm,
                                          const DevCtl& ctl) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, &sm.abort, ctl));
}

struct KvTile {
  int src;       // 0: k/v (prefill keys or suffix keys), 1: cached prefix
  int tile;
  bool partial;
  bool any_fast;
  bool any_pad;
};

// Cached tiles are partial when ragged or when the cache has a validity mask.
template <bool kSuffix>
__device__ __forceinline__ KvTile kv_tile_at(const uint16_t* list, int idx, int n_cache, int P,
                                             bool cache_masked) {
  if (kSuffix && idx < n_cache)
    return KvTile{1, idx, cache_masked || (idx + 1) * kBN > P, false, false};
  const uint16_t e = list[kSuffix ? idx - n_cache : idx];
  return KvTile{0, (int)(e & kTileIndex), (e & kTilePartial) != 0, (e & kTileAnyFast) != 0,
                (e & kTileAnyPad) != 0};
}

// One work unit: a (batch, pair tile, key split) triple, plus its key range.
struct Unit {
  int b, pair, split;
  int tq0, tq1;        // first / last valid query token of the pair tile
  int it_begin, n_it;  // this split's slice of the visited key tiles
  int piece;           // prefill tail split: the piece's index, else -1
};

// Warp-collective: classifies every key tile for the unit's query tokens
// [tq0, tq1] and writes the visited ones, in order, to `list`:
//   skip    no query of the unit sees any key of the tile
//   full    every query sees every key (no per-element predicate)
//   partial per-row visible prefix, FAST hole for expert rows
// Returns the number of entries (the same in every lane).
template <class SmemT>
__device__ int build_tile_list(const SmemT& sm, const uint16_t* codes, int tq0, int tq1,
                               int n_key_tok, uint16_t* list, int lane) {
  const int n_ktiles = (n_key_tok + kBN - 1) / kBN;
  int any_e = 0, all_e = 1;
  for (int t = tq0 + lane; t <= tq1; t += 32) {
    const int e = (codes[t] >> 1) & 1;
    any_e |= e;
    all_e &= e;
  }
  any_e = __any_sync(0xffffffffu, any_e);
  all_e = __all_sync(0xffffffffu, all_e);
  const uint32_t csq0 = codes[tq0] >> 2, csq1 = codes[tq1] >> 2;
  int base = 0;
  for (int t0 = 0; t0 < n_ktiles; t0 += 32) {
    const int t = t0 + lane;
    int c = 0;
    bool any_f = false;
    bool any_p = false;
    if (t < n_ktiles) {
      const uint32_t csk0 = sm.tile_cs_first[t], csk1 = sm.tile_cs_last[t];
      const uint32_t fl = sm.tile_fast[t];
      any_f = (fl & 1) != 0;
      const bool all_f = (fl & 2) != 0;
      any_p = (fl & 4) != 0;
      const bool all_p = (fl & 8) != 0;
      const bool complete = (t + 1) * kBN <= n_key_tok;
      if (csk0 > csq1 || (all_e && all_f) || all_p) c = 0;
      else if (csk1 <= csq0 && !(any_e && any_f) && !any_p && complete) c = 1;
      else c = 2;
    }
    const unsigned m = __ballot_sync(0xffffffffu, c != 0);
    if (c != 0 && list != nullptr) {
      const int pos = base + __popc(m & ((1u << lane) - 1));
      list[pos] = (uint16_t)(t | (c == 2 ? kTilePartial : 0) | (any_f ? kTileAnyFast : 0) |
                             (any_p ? kTileAnyPad : 0));
    }
    base += __popc(m);
  }
  __syncwarp();
  return base;
}

// Warp-collective: the unit with index u and this warp's tile list for it.
// Not inlined: every warp role calls it, and one copy keeps the kernel's code
// (which far exceeds an SM's instruction cache) smaller.
template <bool kSuffix, class SmemT>
__device__ __noinline__ Unit make_unit(int u, const TcParams& p, int n_pairs, int n_cache,
                                          const SmemT& sm, const uint16_t* codes, uint16_t* list,
                                          int lane) {
  Unit x;
  int splits = p.n_splits, t;
  if (!kSuffix && u >= p.n_main) {
    // A tail unit: piece u - n_main of the units after the full rounds.
    const int v = u - p.n_main;
    splits = p.tail_splits;
    x.split = v % splits;
    t = p.n_main + v / splits;
    x.piece = v;
  } else {
    x.split = u % p.n_splits;
    t = u / p.n_splits;
    x.piece = -1;
  }
  x.pair = t % n_pairs;
  x.b = t / n_pairs;
  const int tok_per_pair = 2 * kBM / p.Hq;
  x.tq0 = x.pair * tok_per_pair;
  x.tq1 = min(x.tq0 + tok_per_pair, p.Sq) - 1;
  int n_list = build_tile_list(sm, codes, x.tq0, x.tq1, p.Sq, list, lane);
  if (p.n_splits == 1 && n_cache + n_list == 0) {
    // Only padding can leave a unit without a key tile (a valid query sees
    // its own token).  Keep one fully masked tile so that every unit of a
    // one-split launch visits a tile and writes its (zero) rows.
    if (list != nullptr && lane == 0) list[0] = (uint16_t)(kTilePartial | kTileAnyPad);
    __syncwarp();
    n_list = 1;
  }
  const int n_total = n_cache + n_list;
  const int per = (n_total + splits - 1) / splits;
  x.it_begin = min(x.split * per, n_total);
  x.n_it = min(x.it_begin + per, n_total) - x.it_begin;
  return x;
}

template <bool kSuffix, bool kCacheMask, class L>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_pair_kernel(const __grid_constant__ TcParams p, const DevCtl ctl, int smem_bytes) {
  using SmemT = Smem<L>;
  constexpr int kK = L::kK, kV = L::kV;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // Both CTAs see the same base offset, so both leave here or neither does.
  if ((int)(smem - smem_raw) + layout_bytes<L>(p.Sq) > smem_bytes || p.Sq > L::kMaxTok) {
    pdl_wait();
    if (threadIdx.x == 0) record_status(ctl, kStatusUnsupported);
    return;
  }
  SmemT& sm = *reinterpret_cast<SmemT*>(smem + L::kOffCtl);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + off_codes<L>());
  uint8_t* sQ = smem + kOffQ;
  uint8_t* kring = smem + kOffRing;
  uint8_t* vring = smem + L::kOffV;
  uint8_t* sP = smem + L::kOffP;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_per_b = p.Sq * p.Hq;
  const int n_pairs = (rows_per_b + 2 * kBM - 1) / (2 * kBM);
  // Prefill: units [0, n_main) whole, then tail_splits pieces of each later one.
  const int n_units = kSuffix ? p.B * n_pairs * p.n_splits
                              : p.n_main + (p.B * n_pairs - p.n_main) * p.tail_splits;
  const int n_tail_pieces = n_units - p.n_main;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int n_key_tok = p.Sq;
  const int n_cache = kSuffix ? (p.P + kBN - 1) / kBN : 0;
  // A separate instantiation carries the cached-key validity mask, so the
  // unmasked suffix pass pays nothing for it.
  constexpr bool cache_masked = kSuffix && kCacheMask;

  // With a batch-shared mask (the persistent case) every unit uses row 0;
  // otherwise this cluster runs exactly one unit and scans that unit's batch
  // row.
  const int b_codes = (cluster / p.n_splits) / n_pairs;
  const uint8_t* ar_b = p.ar + (long long)b_codes * p.mask_bs;
  const int32_t* seg_b = p.seg ? p.seg + (long long)b_codes * p.mask_bs : nullptr;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kK; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kV; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 8);
    }
    mbar_init(&sm.p_full, 8);
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.o_free, 8);
    mbar_init(&sm.drain_qk, 1);
    mbar_init(&sm.drain_pv, 1);
    sm.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_q);
    tma_prefetch_desc(&p.map_k);
    tma_prefetch_desc(&p.map_vh);
    tma_prefetch_desc(&p.map_o);
    if (kSuffix) {
      tma_prefetch_desc(&p.map_kc);
      tma_prefetch_desc(&p.map_vch);
    }
  }
  // Both CTAs' barriers must exist before either side signals the other.
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  // Everything above touches no global memory, so it may overlap the previous
  // kernel in the stream; from here on its results are visible.
  pdl_wait();
  pdl_launch_dependents();
  // The mask bytes are the first global reads; their latency hides behind
  // the early TMA issue below.
  const Flags32 flags0 = load_flags32(ar_b, seg_b, n_key_tok, (int)threadIdx.x * 32);
  // With a single split every unit visits at least one key tile (a valid
  // query sees its own token; a unit of padding rows gets one masked tile),
  // so the first unit's Q can load during the mask scan.
  // Without segment ids (or in a suffix pass with a cache, whose cached tiles
  // come first) the unit's first key tile is also known: tile 0, since every
  // query sees key 0 by the block-index rule.  Its K and V then load during the
  // scan as well.  (Segment ids can hide tile 0 -- FAST keys from expert rows,
  // padding -- so those launches wait for the scan.)
  const bool early_q = p.n_splits == 1;
  const bool early_kv = early_q && (p.seg == nullptr || (kSuffix && p.P > 0));
  if (early_q && threadIdx.x == 0) {
    const int pair0 = cluster % n_pairs, b0 = cluster / n_pairs;
    if (leader) mbar_arrive_expect_tx(&sm.q_full, 2 * kQBytes);
    tma_load_4d_pair(sQ, &p.map_q, mapa_shared(smem_u32(&sm.q_full), 0), 0,
                     pair0 * 2 * kBM + (int)rank * kBM, 0, b0);
  }
  if (early_kv && threadIdx.x == 0) {
    const int b0 = cluster / n_pairs;
    if (leader) {
      mbar_arrive_expect_tx(&sm.k_full[0], 2 * kKItem);
      mbar_arrive_expect_tx(&sm.v_full[0], 2 * kVItem);
      mbar_arrive_expect_tx(&sm.v_full[1], 2 * kVItem);
    }
    const bool cache0 = kSuffix && p.P > 0;
    const CUtensorMap* mk = cache0 ? &p.map_kc : &p.map_k;
    const CUtensorMap* mv = cache0 ? &p.map_vch : &p.map_vh;
    tma_load_4d_pair(kring, mk, mapa_shared(smem_u32(&sm.k_full[0]), 0), 0, 64 * (int)rank, 0,
                     b0);
    tma_load_4d_pair(vring, mv, mapa_shared(smem_u32(&sm.v_full[0]), 0), 0, 0, 2 * (int)rank,
                     b0);
    tma_load_4d_pair(vring + kVItem, mv, mapa_shared(smem_u32(&sm.v_full[1]), 0), 0, 64,
                     2 * (int)rank, b0);
  }
  build_codes_x32<kThreads>(ar_b, seg_b, n_key_tok, pad_tokens(n_key_tok), codes, sm.scan,
                            flags0, TileSums{sm.tile_cs_first, sm.tile_cs_last, sm.tile_fast});
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sm.tmem_base;
  const uint32_t tO = tmem + kColO;
  const uint32_t tS = tmem + kColS;      // S[b] at +128*b
  // Warps 1 and 6 (the MMA issuers) only need the tile count.
  uint16_t* list = (warp == 0 || (warp >= 2 && warp <= 5)) ? sm.list[warp] : nullptr;

  if (warp == 0) {
    // ------------------------------------------------- producer (both CTAs)
    // Per unit: Q, then K0, K1, and for each tile j: K(j+2), V(j) keys 0-63,
    // V(j) keys 64-127.  Each ring is filled and consumed in order.
    const uint32_t q_full_l = mapa_shared(smem_u32(&sm.q_full), 0);
    uint32_t uk = 0, uv = 0;        // K / V items issued
    uint32_t nq = 0;                // Q loads issued
    bool ok = true;
    for (int unit = cluster; unit < n_units && ok; unit += n_clusters) {
      const Unit x = make_unit<kSuffix>(unit, p, n_pairs, n_cache, sm, codes, list, lane);
      if (x.n_it == 0) continue;
      const int row0 = x.pair * 2 * kBM + (int)rank * kBM;
      if (nq > 0 || !early_q) {      // else the first Q was issued before the scan
        if (nq > 0 && !warp_wait(&sm.q_empty, (nq - 1) & 1, sm, ctl)) break;
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&sm.q_full, 2 * kQBytes);
          tma_load_4d_pair(sQ, &p.map_q, q_full_l, 0, row0, 0, x.b);
        }
        __syncwarp();
      }
      const bool first_unit = nq == 0;
      ++nq;
      auto load_k = [&](int idx) -> bool {
        const KvTile kt = kv_tile_at<kSuffix>(list, idx, n_cache, p.P, cache_masked);
        const int s = (int)(uk % kK);
        const uint32_t rel = uk / kK;
        if (early_kv && first_unit && uk == 0) {  // tile 0's K was issued before the scan
          ++uk;
          return true;
        }
        if (rel > 0 && !warp_wait(&sm.k_empty[s], (rel - 1) & 1, sm, ctl)) return false;
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&sm.k_full[s], 2 * kKItem);
          // this CTA's 64 keys of the tile, all 256 columns
          tma_load_4d_pair(kring + s * kKItem, kt.src ? &p.map_kc : &p.map_k,
                           mapa_shared(smem_u32(&sm.k_full[s]), 0), 0,
                           kt.tile * kBN + 64 * (int)rank, 0, x.b);
        }
        __syncwarp();
        ++uk;
        return true;
      };
      auto load_v = [&](int idx, int h) -> bool {
        const KvTile kt = kv_tile_at<kSuffix>(list, idx, n_cache, p.P, cache_masked);
        const int s = (int)(uv % kV);
        const uint32_t rel = uv / kV;
        if (early_kv && first_unit && uv < 2) {   // tile 0's V was issued before the scan
          ++uv;
          return true;
        }
        if (rel > 0 && !warp_wait(&sm.v_empty[s], (rel - 1) & 1, sm, ctl)) return false;
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&sm.v_full[s], 2 * kVItem);
          // keys [64h, 64h + 64) of the tile, this CTA's 128 columns
          tma_load_4d_pair(vring + s * kVItem, kt.src ? &p.map_vch : &p.map_vh,
                           mapa_shared(smem_u32(&sm.v_full[s]), 0), 0, kt.tile * kBN + 64 * h,
                           2 * (int)rank, x.b);
        }
        __syncwarp();
        ++uv;
        return true;
      };
      const int i0 = x.it_begin, n = x.n_it;
      ok = load_k(i0);
      if (ok && n > 1) ok = load_k(i0 + 1);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 2 < n) ok = load_k(i0 + j + 2);
        if (ok) ok = load_v(i0 + j, 0);
        if (ok) ok = load_v(i0 + j, 1);
      }
    }
    // Every load completes on the even CTA's barriers: there, wait (bounded)
    // for the last phase of each, so no copy into either CTA is still in
    // flight when the cluster leaves.  Phases the consumer already waited for
    // return at once.
    if (leader && lane == 0) {
      if (nq > 0) (void)mbar_wait(&sm.q_full, (nq - 1) & 1, ctl);
      for (int s = 0; s < kK; ++s) {
        const uint32_t n_s = uk > (uint32_t)s ? (uk - (uint32_t)s + kK - 1) / kK : 0;
        if (n_s > 0) (void)mbar_wait(&sm.k_full[s], (n_s - 1) & 1, ctl);
      }
      for (int s = 0; s < kV; ++s) {
        const uint32_t n_s = uv > (uint32_t)s ? (uv - (uint32_t)s + kV - 1) / kV : 0;
        if (n_s > 0) (void)mbar_wait(&sm.v_full[s], (n_s - 1) & 1, ctl);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 6) {
    // ------------------------- MMA issuers (even CTA only): QK by warp 1, PV by warp 6
    // Two issuing threads, so a PV that waits for its P never holds back the
    // QK of a later tile and vice versa.  Each accumulation chain (S of one
    // tile, O of one unit) and each ring belongs to one thread: tcgen05
    // ordering and commit tracking are per thread.
    if (leader) {
      auto commit_both = [&](uint64_t* bar) {
        umma_commit_pair(mapa_shared(smem_u32(bar), 0));
        umma_commit_pair(mapa_shared(smem_u32(bar), 1));
      };
      uint32_t g = 0;     // key tiles processed, across units
      uint32_t nu = 0;    // units started
      bool ok = true;
      if (warp == 1) {
        const uint64_t qdesc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t kdesc0 = sdesc_sw128(smem_u32(kring), 16, 1024);
        uint32_t uk = 0;
        for (int unit = cluster; unit < n_units && ok; unit += n_clusters) {
          const Unit x = make_unit<kSuffix>(unit, p, n_pairs, n_cache, sm, codes, list, lane);
          if (x.n_it == 0) continue;
          if (!warp_wait(&sm.q_full, nu & 1, sm, ctl)) break;
          ++nu;
          for (int j = 0; j < x.n_it; ++j) {
            const uint32_t gi = g + (uint32_t)j;
            const int s = (int)(uk % kK);
            if (!warp_wait(&sm.k_full[s], (uk / kK) & 1, sm, ctl)) { ok = false; break; }
            // S[gi%2] was last read by the softmax of tile gi-2.
            if (gi >= 2 && !warp_wait(&sm.s_free[gi & 1], ((gi - 2) >> 1) & 1, sm, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (lane == 0) {
              const uint64_t kd = kdesc0 + (uint64_t)((s * kKItem) >> 4);
#pragma unroll
              for (int kk = 0; kk < kD / 16; ++kk) {
                // A = Q[128 rows per CTA x 16 d], B = K[64 keys per CTA x 16 d],
                // both K-major: 8-row groups 1024 B apart; the K step walks
                // 32 B inside a 64-column block, then the next block.
                const uint32_t qoff = (uint32_t)((kk >> 2) * kQBlk + (kk & 3) * 32);
                const uint32_t koff = (uint32_t)((kk >> 2) * kKBlk + (kk & 3) * 32);
                umma_pair_ss(tS + 128 * (gi & 1), qdesc0 + (uint64_t)(qoff >> 4),
                             kd + (uint64_t)(koff >> 4), kIdescQK, kk > 0 ? 1u : 0u);
              }
              commit_both(&sm.k_empty[s]);
              commit_both(&sm.s_full[gi & 1]);
              if (j == x.n_it - 1) commit_both(&sm.q_empty);   // the unit's last QK read Q
            }
            __syncwarp();
            ++uk;
          }
          g += (uint32_t)x.n_it;
        }
        if (lane == 0) umma_commit_pair(smem_u32(&sm.drain_qk));
        __syncwarp();
        (void)mbar_wait(&sm.drain_qk, 0, ctl);
      } else {
        const uint64_t pdesc0 = sdesc_sw128(smem_u32(sP), 16, 1024);
        const uint64_t vdesc0 = sdesc_sw128(smem_u32(vring), kVBlk, 1024);
        uint32_t uv = 0;
        for (int unit = cluster; unit < n_units && ok; unit += n_clusters) {
          const Unit x = make_unit<kSuffix>(unit, p, n_pairs, n_cache, sm, codes, list, lane);
          if (x.n_it == 0) continue;
          ++nu;
          for (int j = 0; j < x.n_it && ok; ++j) {
            const uint32_t gi = g + (uint32_t)j;
            // V arrives long before P: wait for it first, off the critical path.
            if (!warp_wait(&sm.v_full[uv % kV], (uv / kV) & 1, sm, ctl)) { ok = false; break; }
            if (!warp_wait(&sm.p_full, gi & 1, sm, ctl)) { ok = false; break; }
            // The unit's first PV overwrites O: the previous unit's epilogue
            // must have read it.
            if (j == 0 && nu > 1 && !warp_wait(&sm.o_free, (nu - 2) & 1, sm, ctl)) {
              ok = false;
              break;
            }
            for (int h = 0; h < 2 && ok; ++h) {
              const int s = (int)(uv % kV);
              if (h == 1 && !warp_wait(&sm.v_full[s], (uv / kV) & 1, sm, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
              if (lane == 0) {
                const uint64_t vd = vdesc0 + (uint64_t)((s * kVItem) >> 4);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                  // A = P[128 rows per CTA x 16 keys], K-major: 8-row groups
                  // 1024 B apart; a K step walks 32 B inside a 64-key block.
                  // B = V[16 keys x (128 columns per CTA)], MN-major: 8-key
                  // groups 1024 B apart, 64-column blocks 8 KB apart; a K
                  // step is 16 rows.
                  const uint32_t poff = (uint32_t)(h * kPBlk + k4 * 32);
                  umma_pair_ss(tO, pdesc0 + (uint64_t)(poff >> 4),
                               vd + (uint64_t)((k4 * 2048) >> 4), kIdescPV,
                               (j > 0 || h > 0 || k4 > 0) ? 1u : 0u);
                }
                commit_both(&sm.v_empty[s]);
                if (h == 1) commit_both(&sm.o_done);
              }
              __syncwarp();
              ++uv;
            }
          }
          g += (uint32_t)x.n_it;
        }
        if (lane == 0) umma_commit_pair(smem_u32(&sm.drain_pv));
        __syncwarp();
        (void)mbar_wait(&sm.drain_pv, 0, ctl);
      }
    }
  } else {
    // ------------------------------------ softmax / epilogue (both CTAs)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // row of this thread in the CTA
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float c = p.scale_log2;                  // > 0
    const uint32_t s_free_l0 = mapa_shared(smem_u32(&sm.s_free[0]), 0);
    const uint32_t s_free_l1 = mapa_shared(smem_u32(&sm.s_free[1]), 0);
    const uint32_t p_full_l = mapa_shared(smem_u32(&sm.p_full), 0);
    const uint32_t o_free_l = mapa_shared(smem_u32(&sm.o_free), 0);
    // This row's 128-byte lines in the two P blocks (K-major, 128-byte swizzle).
    uint8_t* const p_row0 = sP + r * 128;
    uint8_t* const p_row1 = sP + kPBlk + r * 128;
    uint32_t g = 0;
    bool store_pending = false;    // this warp's output stores may still read P
    bool ok = true;

    // The next unit's tile list is built while the current unit's last PV
    // runs (the list of the current unit is no longer read then).
    Unit nx = make_unit<kSuffix>(cluster, p, n_pairs, n_cache, sm, codes, list, lane);
    for (int unit = cluster; unit < n_units && ok; unit += n_clusters) {
      const Unit x = nx;
      const int row0 = x.pair * 2 * kBM + (int)rank * kBM;
      const bool row_valid = row0 + r < rows_per_b;
      // Where a partial result of this row goes: split-K over the cache
      // (suffix: [split][batch][row]) or a prefill tail piece ([piece][256
      // rows]); unnormalised O rows, then (m, l) pairs.
      float* po = nullptr;
      float* pml = nullptr;
      if (p.n_splits > 1) {
        const long long slot = ((long long)x.split * p.B + x.b) * rows_per_b + row0 + r;
        po = p.ws + slot * kD;
        pml = p.ws + (long long)p.n_splits * p.B * rows_per_b * kD + slot * 2;
      } else if (x.piece >= 0) {
        const long long ts = (long long)x.piece * (2 * kBM) + (int)rank * kBM + r;
        po = p.ws + ts * kD;
        pml = p.ws + (long long)n_tail_pieces * (2 * kBM) * kD + ts * 2;
      }
      if (x.n_it == 0) {
        if (pml != nullptr && row_valid) {
          pml[0] = -INFINITY;
          pml[1] = 0.f;
        }
        if (unit + n_clusters < n_units)
          nx = make_unit<kSuffix>(unit + n_clusters, p, n_pairs, n_cache, sm, codes, list, lane);
        continue;
      }
      const int tok = min(x.tq0 + ((int)rank * kBM + r) / p.Hq, x.tq1);
      const uint32_t cq = codes[tok];
      const uint32_t csq = cq >> 2;
      const bool row_expert = (cq & 2u) != 0;
      const bool row_pad = is_pad(cq);               // a padding query sees nothing
      float m_run = -INFINITY;
      float l_run = 0.f;

      for (int li = 0; li < x.n_it; ++li) {
        const uint32_t gi = g + (uint32_t)li;
        const int bs = (int)(gi & 1);
        const KvTile kt = kv_tile_at<kSuffix>(list, x.it_begin + li, n_cache, p.P, cache_masked);
        // Validity bytes of a cached tile, loaded before the wait for S: byte
        // lane + 32w of the tile in v[w].
        uint32_t vraw[4] = {0u, 0u, 0u, 0u};
        if (kSuffix && kt.src == 1 && cache_masked) {
          const uint8_t* cv = p.cache_valid + (long long)x.b * p.P + kt.tile * kBN;
          const int n_here = min(kBN, p.P - kt.tile * kBN);
#pragma unroll
          for (int w = 0; w < 4; ++w)
            vraw[w] = (lane + 32 * w < n_here) ? (uint32_t)cv[lane + 32 * w] : 0u;
        }
        if (!warp_wait(&sm.s_full[bs], (gi >> 1) & 1, sm, ctl)) { ok = false; break; }
        tc_fence_after();
        float xs[kBN];
        {
          // all four 32-column loads in flight, one wait
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tS + lane_off + 128 * bs, r0);
          tmem_ld32(tS + lane_off + 128 * bs + 32, r1);
          tmem_ld32(tS + lane_off + 128 * bs + 64, r2);
          tmem_ld32(tS + lane_off + 128 * bs + 96, r3);
          tmem_ld_wait();
          reg_fence(r0);
          reg_fence(r1);
          reg_fence(r2);
          reg_fence(r3);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            xs[e] = __uint_as_float(r0[e]);
            xs[32 + e] = __uint_as_float(r1[e]);
            xs[64 + e] = __uint_as_float(r2[e]);
            xs[96 + e] = __uint_as_float(r3[e]);
          }
        }
        // S is in registers: the next QK into this buffer may start.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(bs ? s_free_l1 : s_free_l0);
        // Partial tiles and padding rows: one 128-bit visibility mask per row
        // (bit j of vm[j / 32] = key j visible), applied in a single pass.
        // The keys a row sees in a partial tile are a prefix (the block index
        // is non-decreasing), minus the FAST keys for expert rows and the
        // padding keys for every row; a cached tile with a validity mask keeps
        // the valid keys of its ragged prefix.
        if (kt.partial || __any_sync(0xffffffffu, row_pad)) {
          uint32_t vm[4] = {~0u, ~0u, ~0u, ~0u};
          if (kt.partial) {
            const int k0 = kt.tile * kBN;
            int e;
            if (kSuffix && kt.src == 1) {
              e = min(kBN, p.P - k0);
              if (cache_masked) {
#pragma unroll
                for (int w = 0; w < 4; ++w) vm[w] = __ballot_sync(0xffffffffu, vraw[w] != 0u);
              }
            } else {
              e = 0;
#pragma unroll
              for (int step = kBN; step >= 1; step >>= 1) {
                const int probe = e + step;
                if (probe <= kBN && (uint32_t)(codes[k0 + probe - 1] >> 2) <= csq) e = probe;
              }
              e = min(e, n_key_tok - k0);
              if (kt.any_fast || kt.any_pad) {
                // FAST bit (padding keys carry it too) and padding, per key.
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                  const uint32_t ck = codes[k0 + 32 * w + lane];
                  const uint32_t fw = __ballot_sync(0xffffffffu, (ck & 1u) != 0u);
                  const uint32_t pw = __ballot_sync(0xffffffffu, is_pad(ck));
                  vm[w] &= ~(row_expert ? fw : pw);
                }
              }
            }
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int lo = 32 * w;
              vm[w] &= e >= lo + 32 ? ~0u : (e <= lo ? 0u : ((1u << (e - lo)) - 1u));
            }
          }
          if (row_pad) vm[0] = vm[1] = vm[2] = vm[3] = 0u;
#pragma unroll
          for (int j = 0; j < kBN; ++j) xs[j] = ((vm[j >> 5] >> (j & 31)) & 1u) ? xs[j] : -INFINITY;
        }
        // Row maximum: eight independent chains of three-input max.
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float a = fmax3(xs[k], xs[k + 8], xs[k + 16]);
#pragma unroll
          for (int i = 3; i < 15; i += 2) a = fmax3(a, xs[k + 8 * i], xs[k + 8 * i + 8]);
          m8[k] = fmaxf(a, xs[k + 120]);
        }
        const float mx =
            fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], fmax3(m8[4], m8[5], m8[6]), m8[7])) * c;

        // Lazy rescaling (exact: O and l always share the reference max).
        const bool upd = mx > m_run + kRescaleThreshold;
        const float m_new = upd ? mx : m_run;
        const float alpha = ex2(m_run - m_new);
        const bool need_o = upd && (m_run != -INFINITY);
        l_run *= (m_run == -INFINITY) ? 0.f : alpha;
        m_run = m_new;
        const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
        const float2 c2 = make_float2(c, c), n2 = make_float2(nm, nm);
        float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        uint32_t pk[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float2 t = ffma2(make_float2(xs[2 * e], xs[2 * e + 1]), c2, n2);
          const float2 pp = make_float2(ex2(t.x), ex2(t.y));
          ls[e & 3] = fadd2(ls[e & 3], pp);
          pk[e] = cvt_bf16x2(pp.x, pp.y);
        }
        const float2 lsum = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
        l_run += lsum.x + lsum.y;

        // PV of the previous tile reads the P buffer and accumulates into O:
        // both must be finished before either is written again.  It has
        // normally finished long before the exponentials above are done.
        if (gi >= 1) {
          if (!warp_wait(&sm.o_done, (gi - 1) & 1, sm, ctl)) { ok = false; break; }
          tc_fence_after();
        }
        if (store_pending) {     // the previous unit's output stores read P
          if (lane == 0) tma_store_wait_read();
          __syncwarp();
          store_pending = false;
        }
        const bool rescale = __any_sync(0xffffffffu, need_o);
        if (rescale) {
          const float a = need_o ? alpha : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < kD / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + lane_off + 32 * cc, o);
            tmem_ld_wait();
            reg_fence(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
            tmem_st32(tO + lane_off + 32 * cc, o);
          }
        }
        // P row -> shared memory: 16-byte chunk j of the row's 128-byte line
        // goes to chunk j ^ (row % 8) (128-byte swizzle, conflict-free).
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int sw = (j ^ (r & 7)) << 4;
          *reinterpret_cast<uint4*>(p_row0 + sw) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          *reinterpret_cast<uint4*>(p_row1 + sw) =
              make_uint4(pk[32 + 4 * j], pk[33 + 4 * j], pk[34 + 4 * j], pk[35 + 4 * j]);
        }
        fence_proxy_async_smem();
        if (rescale) tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(p_full_l);
      }
      if (!ok) break;

      // ------------------------------------------------------- epilogue
      const uint32_t g_last = g + (uint32_t)x.n_it - 1;
      g += (uint32_t)x.n_it;
      if (unit + n_clusters < n_units)
        nx = make_unit<kSuffix>(unit + n_clusters, p, n_pairs, n_cache, sm, codes, list, lane);
      if (!warp_wait(&sm.o_done, g_last & 1, sm, ctl)) { ok = false; break; }
      tc_fence_after();
      const long long grow = (long long)x.b * rows_per_b + row0 + r;
      if (po == nullptr) {
        // A row that saw no key (a padding query) writes 0, lse = -inf.
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        // The P buffer is free once the last PV has finished: each warp stages
        // its own 32 rows there, 64 columns per 4 KB swizzled box, in two
        // rounds of two boxes.
        uint8_t* const st0 = sP + quarter * 4096;
        uint8_t* const st1 = sP + kPBlk + quarter * 4096;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          if (half == 1) {
            if (lane == 0) tma_store_wait_read();
            __syncwarp();
          }
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const int col = 128 * half + 64 * sub;
            uint32_t o0[32], o1[32];
            tmem_ld32(tO + lane_off + col, o0);
            tmem_ld32(tO + lane_off + col + 32, o1);
            tmem_ld_wait();
            reg_fence(o0);
            reg_fence(o1);
            uint32_t ob[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              ob[e] = cvt_bf16x2(__uint_as_float(o0[2 * e]) * inv,
                                 __uint_as_float(o0[2 * e + 1]) * inv);
              ob[16 + e] = cvt_bf16x2(__uint_as_float(o1[2 * e]) * inv,
                                      __uint_as_float(o1[2 * e + 1]) * inv);
            }
            uint8_t* line = (sub ? st1 : st0) + lane * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(line + ((j ^ (lane & 7)) << 4)) =
                  make_uint4(ob[4 * j], ob[4 * j + 1], ob[4 * j + 2], ob[4 * j + 3]);
          }
          if (half == 1) {
            // All of O has been read: the next unit's first PV may overwrite it.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(o_free_l);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_4d(&p.map_o, st0, 0, row0 + quarter * kStageRows, 2 * half, x.b);
            tma_store_4d(&p.map_o, st1, 0, row0 + quarter * kStageRows, 2 * half + 1, x.b);
            tma_store_commit();
          }
          __syncwarp();
        }
        store_pending = true;
        if (!kSuffix && p.lse && row_valid)
          p.lse[grow] = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      } else {
        // Split partial: unnormalised O and (m, l) for a combine kernel.
        // tcgen05.ld is warp-collective (.sync.aligned): every lane loads,
        // only lanes holding a real row store.
        float* wo = po;
#pragma unroll 1
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * cc, o);
          tmem_ld_wait();
          reg_fence(o);
          if (row_valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(wo + 32 * cc + e) =
                  make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                              __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(o_free_l);
        if (row_valid) {
          pml[0] = m_run;
          pml[1] = l_run;
        }
      }
    }
    if (store_pending && lane == 0) tma_store_wait_read();
    __syncwarp();
  }

  // Neither CTA may leave while its partner can still signal its barriers or
  // read its shared memory; then both free their TMEM.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Merges split-K partials: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// with M = max_s m_s (the log-sum-exp rule).  One warp per output row; each
// lane handles 8 of the 256 columns.  HBM-bound: it reads the fp32 partials
// once and writes the bf16 row once.
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ ws, __nv_bfloat16* __restrict__ out, int n_splits,
                   long long n_rows) {
  pdl_wait();                  // the partials come from the kernel before
  pdl_launch_dependents();
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const float* ml = ws + (long long)n_splits * n_rows * kD;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ml[(s * n_rows + row) * 2]);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float L = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float m = ml[(s * n_rows + row) * 2];
    const float l = ml[(s * n_rows + row) * 2 + 1];
    if (l == 0.f) continue;
    const float w = ex2(m - M);
    L += w * l;
    const float4* src = reinterpret_cast<const float4*>(ws + (s * n_rows + row) * kD + lane * 8);
    const float4 a = src[0], c = src[1];
    acc[0] += w * a.x; acc[1] += w * a.y; acc[2] += w * a.z; acc[3] += w * a.w;
    acc[4] += w * c.x; acc[5] += w * c.y; acc[6] += w * c.z; acc[7] += w * c.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;   // every split empty: a padding row
  uint4 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + row * kD + lane * 8) = pk;
}

// Merges the prefill tail pieces: for each row of a tail unit (units from
// n_main on, each split into `splits` pieces over its key tiles), out = sum_k
// 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k with M = max_k m_k (the log-sum-exp
// rule), and lse.  One warp per row, 8 columns per lane; pieces with l = 0
// (no visible key) drop out; a row with none writes 0 and lse = -inf.
__global__ void __launch_bounds__(256)
    tail_combine_kernel(const float* __restrict__ ws, __nv_bfloat16* __restrict__ out,
                        float* __restrict__ lse, int n_main, int n_tail_units, int splits,
                        int n_pairs, int rows_per_b) {
  pdl_wait();                  // the partials come from the kernel before
  pdl_launch_dependents();
  const long long tr = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);   // tail row
  const int lane = threadIdx.x & 31;
  if (tr >= (long long)n_tail_units * 2 * kBM) return;
  const int unit = n_main + (int)(tr / (2 * kBM));
  const int rr = (int)(tr % (2 * kBM));                // row of the 256-row tile
  const int b = unit / n_pairs, pair = unit % n_pairs;
  const int row = pair * 2 * kBM + rr;
  if (row >= rows_per_b) return;
  const long long n_rows_ws = (long long)n_tail_units * splits * 2 * kBM;
  const long long ts0 = (long long)(unit - n_main) * splits * 2 * kBM + rr;  // piece 0's row
  const float2* ml = reinterpret_cast<const float2*>(ws + n_rows_ws * kD);
  float M = -INFINITY;
  for (int k = 0; k < splits; ++k) {
    const float2 v = ml[ts0 + (long long)k * 2 * kBM];
    if (v.y > 0.f) M = fmaxf(M, v.x);
  }
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float L = 0.f;
  for (int k = 0; k < splits; ++k) {
    const long long ts = ts0 + (long long)k * 2 * kBM;
    const float2 v = ml[ts];
    if (v.y <= 0.f) continue;
    const float w = ex2(v.x - M);
    L += w * v.y;
    const float4* src = reinterpret_cast<const float4*>(ws + ts * kD + lane * 8);
    const float4 a = src[0], c = src[1];
    acc[0] += w * a.x; acc[1] += w * a.y; acc[2] += w * a.z; acc[3] += w * a.w;
    acc[4] += w * c.x; acc[5] += w * c.y; acc[6] += w * c.z; acc[7] += w * c.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint4 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  const long long grow = (long long)b * rows_per_b + row;
  *reinterpret_cast<uint4*>(out + grow * kD + lane * 8) = pk;
  if (lse != nullptr && lane == 0)
    lse[grow] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// Dynamic shared memory for S code tokens: the layout plus up to 1 KB to
// align its base, capped at the per-CTA limit (the kernel checks that its
// aligned layout fits what it was given).
template <class L>
int pair_smem_bytes(int n_code_tokens) {
  return min(layout_bytes<L>(n_code_tokens) + 1024, kSmemLimit);
}

template <bool kSuffix, bool kCacheMask, class L>
cudaError_t launch_pair(const TcParams& p, const DevCtl& ctl, dim3 grid, cudaStream_t st) {
  // Per call: the attribute belongs to the device (and to the module, which a
  // device reset reloads).
  const cudaError_t attr_err = cudaFuncSetAttribute(
      tc_pair_kernel<kSuffix, kCacheMask, L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      kSmemLimit);
  if (attr_err != cudaSuccess) return attr_err;
  const int smem = pair_smem_bytes<L>(p.Sq);
  return launch_pdl(tc_pair_kernel<kSuffix, kCacheMask, L>, grid, dim3(kThreads), smem, st, p,
                    ctl, smem);
}

template <class L>
cudaError_t launch_mode(const TcParams& p, bool suffix_mode, const DevCtl& ctl, dim3 grid,
                        cudaStream_t st) {
  if (!suffix_mode) return launch_pair<false, false, L>(p, ctl, grid, st);
  return p.cache_valid ? launch_pair<true, true, L>(p, ctl, grid, st)
                       : launch_pair<true, false, L>(p, ctl, grid, st);
}

// The tile classes build_tile_list gives, exported for tests: one CTA per
// (256-row tile, batch element) scans the mask like the attention kernel and
// writes out[b][pair][key tile] = 0 (skipped), 1 (full) or 2 (partial).
struct DbgTileSmem {
  int scan[kThreads / 32];
  uint16_t list[kMaxTokens / kBN + 2];
  uint16_t tile_cs_first[kMaxTokens / kBN + 2];
  uint16_t tile_cs_last[kMaxTokens / kBN + 2];
  uint8_t tile_fast[kMaxTokens / kBN + 2];
};

__global__ void __launch_bounds__(kThreads)
    debug_tiles_kernel(const uint8_t* ar, const int32_t* seg, long long mask_bs, int S, int Hq,
                       uint8_t* out) {
  extern __shared__ __align__(16) uint8_t dbg_raw[];
  DbgTileSmem& sm = *reinterpret_cast<DbgTileSmem*>(dbg_raw);
  uint16_t* codes = reinterpret_cast<uint16_t*>(dbg_raw + ((sizeof(DbgTileSmem) + 127) / 128) * 128);
  const int pair = blockIdx.x, b = blockIdx.y, n_pairs = gridDim.x;
  const int n_kt = (S + kBN - 1) / kBN;
  const uint8_t* ar_b = ar + (long long)b * mask_bs;
  const int32_t* seg_b = seg ? seg + (long long)b * mask_bs : nullptr;
  const Flags32 f0 = load_flags32(ar_b, seg_b, S, (int)threadIdx.x * 32);
  build_codes_x32<kThreads>(ar_b, seg_b, S, pad_tokens(S), codes, sm.scan, f0,
                            TileSums{sm.tile_cs_first, sm.tile_cs_last, sm.tile_fast});
  uint8_t* o = out + ((long long)b * n_pairs + pair) * n_kt;
  for (int t = threadIdx.x; t < n_kt; t += blockDim.x) o[t] = 0;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int tok_per_pair = 2 * kBM / Hq;
    const int tq0 = pair * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
    const int n = build_tile_list(sm, codes, tq0, tq1, S, sm.list, lane);
    for (int i = lane; i < n; i += 32) {
      const uint16_t e = sm.list[i];
      o[e & kTileIndex] = (e & kTilePartial) ? 2 : 1;
    }
  }
}

}  // namespace

cudaError_t launch_debug_tiles(const uint8_t* ar, const int32_t* seg, long long mask_bs, int B,
                               int S, int Hq, uint8_t* out, cudaStream_t st) {
  const int n_pairs = (S * Hq + 2 * kBM - 1) / (2 * kBM);
  const int smem = (int)((sizeof(DbgTileSmem) + 127) / 128 * 128) + pad_tokens(S) * 2;
  const cudaError_t attr = cudaFuncSetAttribute(
      debug_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  if (attr != cudaSuccess) return attr;
  debug_tiles_kernel<<<dim3(n_pairs, B), kThreads, smem, st>>>(ar, seg, mask_bs, S, Hq, out);
  return cudaGetLastError();
}

// SM count of the current device, looked up once per device (a process may
// drive GPUs with different counts).
int sm_count() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < kMaxDev) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  if (dev < kMaxDev) cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

cudaError_t launch_tc_pair(const TcParams& p, bool suffix_mode, const DevCtl& ctl,
                           cudaStream_t st) {
  const int rows = p.Sq * p.Hq;
  const int n_pairs = (rows + 2 * kBM - 1) / (2 * kBM);
  const int n_whole = p.B * n_pairs * p.n_splits;
  const int n_slots = max(sm_count() / 2, 1);
  TcParams q = p;
  q.n_main = n_whole;
  q.tail_splits = 1;
  if (!suffix_mode && p.mask_bs == 0 && p.ws != nullptr && p.n_splits == 1) {
    q.tail_splits = tc_prefill_tail_splits(p.B, p.Sq, p.Hq);
    if (q.tail_splits > 1) q.n_main = n_whole / n_slots * n_slots;
  }
  const int n_units = q.n_main + (n_whole - q.n_main) * q.tail_splits;
  // A batch-shared mask lets one cluster per SM pair walk many units;
  // per-batch masks get one cluster per unit (each scans its own row).
  const int n_clusters = p.mask_bs == 0 ? min(n_units, n_slots) : n_units;
  dim3 grid(2 * n_clusters, 1);
  const bool short_s = p.Sq <= LayoutShort::kMaxTok;
  cudaError_t e = short_s ? launch_mode<LayoutShort>(q, suffix_mode, ctl, grid, st)
                          : launch_mode<LayoutLong>(q, suffix_mode, ctl, grid, st);
  if (e != cudaSuccess) return e;
  if (q.tail_splits > 1) {
    const int n_tail = n_whole - q.n_main;
    const long long n_rows = (long long)n_tail * 2 * kBM;
    return launch_pdl(tail_combine_kernel, dim3((unsigned)((n_rows + 7) / 8)), dim3(256), 0, st,
                      static_cast<const float*>(p.ws),
                      reinterpret_cast<__nv_bfloat16*>(p.out_ptr), p.lse, q.n_main, n_tail,
                      q.tail_splits, n_pairs, rows);
  }
  if (p.n_splits <= 1) return e;
  const long long n_rows = (long long)p.B * rows;
  return launch_pdl(combine_kernel, dim3((unsigned)((n_rows + 7) / 8)), dim3(256), 0, st,
                    static_cast<const float*>(p.ws), reinterpret_cast<__nv_bfloat16*>(p.out_ptr),
                    p.n_splits, n_rows);
}

cudaError_t launch_combine(const float* ws, __nv_bfloat16* out, int n_splits, long long n_rows,
                           cudaStream_t st) {
  return launch_pdl(combine_kernel, dim3((unsigned)((n_rows + 7) / 8)), dim3(256), 0, st, ws, out,
                    n_splits, n_rows);
}

int tc_suffix_splits(int B, int Sq, int P, int Hq) {
  // Split the key tiles over several CTA pairs only when the pairs of one
  // split would leave SMs idle: enough splits to fill the SMs once, each
  // keeping at least two key tiles, at most 8.
  const int rows = Sq * Hq;
  const int n_ctas = 2 * ((rows + 2 * kBM - 1) / (2 * kBM)) * B;
  const int tiles = (P + kBN - 1) / kBN + (Sq + kBN - 1) / kBN;
  int s = sm_count() / max(n_ctas, 1);
  s = min(s, tiles / 2);
  s = min(s, 8);
  return max(s, 1);
}

int tc_prefill_tail_splits(int B, int Sq, int Hq) {
  // When the last round of whole units would leave at least half the SM
  // pairs idle, the full rounds run whole and each remaining unit is split
  // over several pairs.  A piece pays a unit's fixed costs (its Q load, a
  // partial write, the merge: about two tiles' time), so it must keep at
  // least 6 key tiles: short sequences (pi0, pi0.5) are left whole, where
  // splitting measured slower.
  const int n_slots = max(sm_count() / 2, 1);
  const int n_whole = B * ((Sq * Hq + 2 * kBM - 1) / (2 * kBM));
  const int full = n_whole / n_slots, rem = n_whole % n_slots;
  if (full < 1 || rem < 1) return 1;
  const int splits = min(min(n_slots / rem, 8), ((Sq + kBN - 1) / kBN) / 6);
  return splits >= 2 ? splits : 1;
}

size_t tc_prefill_tail_bytes() {
  // At most one round of pieces, one per SM pair, of 256 rows.
  const size_t pieces = (size_t)max(sm_count() / 2, 1);
  return pieces * 2 * kBM * (kD + 2) * sizeof(float);
}

size_t tc_suffix_workspace_bytes(int B, int Sq, int P, int Hq) {
  const int s = tc_suffix_splits(B, Sq, P, Hq);
  if (s <= 1) return 0;
  const size_t rows = (size_t)B * Sq * Hq;
  return (size_t)s * rows * (kD + 2) * sizeof(float);
}

}  // namespace piattn
