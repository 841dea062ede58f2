// tc_attention.cu -- bf16 joint (prefix-LM) attention on tcgen05 tensor cores.
//
// One CTA computes one 128-row query tile: 128 / Hq query tokens x Hq heads.
// In the token-major [B, S, Hq, 256] layout those rows are contiguous, and
// with a single KV head they all read the same K/V rows, so every K/V tile
// brought into shared memory serves all heads ("π0.5 vs MM-DiT joint
// attention", "joint attention 只管算子": 8 query heads, 1 KV head, head_dim
// 256, one shared KV pool).
//
// Per key tile of 64 keys:
//   S  = Q K^T     tcgen05.mma kind::f16, A = Q (TMEM), B = K (smem), D in TMEM
//   P  = exp2(S * scale*log2e - m)   fp32 online softmax, one thread per row
//   O += P V       tcgen05.mma, A = P (TMEM, bf16), B = V (smem, MN-major)
// Both MMAs take A from tensor memory, so shared memory only carries K and V:
// a 6-deep ring of 32 KB tiles keeps several loads in flight.
//
// The mask is evaluated in-kernel from the packed per-token codes of
// mask.cuh: key tiles no query of the tile can see are never loaded, tiles
// every query sees in full skip the predicate, and in the others each row
// keeps the keys below its visible-prefix length (the cumsum rule makes the
// visible keys of a tile a prefix of it) minus, for expert rows, FAST keys.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Q once, then K/V tiles through the ring
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..5  Q -> TMEM, softmax, O correction and the epilogue; warp w
//               owns TMEM lanes / tile rows 32*(w%4) .. 32*(w%4)+31
//
// TMEM (512 columns): O fp32 [0,256) | Q bf16 [256,384) | S0 [384,448) |
// S1 [448,512).  P of tile t is written as packed bf16 over the first 32
// columns of S[t%2].
//
// Shared memory: ring 6 x 32 KB | control block | per-token codes.  Q is
// staged through ring stages 0-1 before it moves to TMEM; the epilogue stages
// the bf16 output there too.  Operand tiles are [rows x 64 bf16] blocks with
// the 128-byte swizzle, as TMA writes them and the UMMA descriptors read them.
// Every tile moves with ONE 4-D TMA instruction whose third dimension walks
// the four 64-column blocks: the TMA engine's per-instruction cost dominates
// for small boxes, and one 32 KB box streams ~30% faster than four 8 KB ones.
//
// Suffix mode ("VLA 代码精读 - OpenPI & StarVLA", 1.6 Pi0.sample_actions): the
// key sequence is the P cached prefix keys followed by the Sq suffix keys; the
// cached keys are visible to every query.  Work can be split over the key
// tiles (split-K); each split then writes unnormalised fp32 partials (O, m, l)
// that a combine kernel merges with the log-sum-exp rule.
//
// Every mbarrier wait is bounded (DevCtl::wait_limit); on expiry the kernel
// records PI_ERR_TIMEOUT, raises a CTA-wide abort flag, drains what it has in
// flight (bounded), frees TMEM and returns.
#include <cfloat>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128;                    // query rows per tile
constexpr int kBN = 64;                     // keys per key tile
constexpr int kD = 256;                     // head dim
constexpr int kBlk = kBN * 128;             // [64 rows x 64 bf16] swizzled block: 8 KB
constexpr int kItemBytes = 4 * kBlk;        // one K or V tile [64 x 256] bf16: 32 KB
constexpr int kStages = 6;
constexpr int kRingBytes = kStages * kItemBytes;
constexpr int kQBlk = kBM * 128;            // [128 rows x 64 bf16]: 16 KB
constexpr int kQStages = (4 * kQBlk) / kItemBytes;  // ring stages Q occupies: 2
constexpr int kMaxKeyTiles = (kMaxTokens + kBN - 1) / kBN + 2;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays <= 256

constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, kD, false, true);

constexpr uint32_t kColO = 0, kColQ = 256, kColS = 384;

// key-tile list entries
constexpr uint16_t kTilePartial = 0x8000;
constexpr uint16_t kTileAnyFast = 0x4000;
constexpr uint16_t kTileIndex = 0x3FFF;

struct __align__(8) Smem {
  uint64_t q_full;               // Q landed in smem (TMA)
  uint64_t q_tmem;               // Q copied into TMEM (softmax warps)
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_list;                    // entries of `list` (prefill: key tiles; suffix: suffix tiles)
  int q_any_exp, q_all_exp;
  uint32_t cq_first, cq_last;
  int scan[kThreads / 32];
  uint16_t list[kMaxKeyTiles];   // tile index | kTilePartial | kTileAnyFast
  uint8_t cls[kMaxKeyTiles];     // 0 skip, 1 full, 2 partial; bit 2: tile has a FAST key
};

constexpr int kOffCtl = kRingBytes;
constexpr int kOffCodes = kOffCtl + ((int)sizeof(Smem) + 127) / 128 * 128;

__host__ __device__ constexpr int pad_tokens(int n) { return (n + 127) / 128 * 128; }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void softmax_bar() {  // the 4 softmax warps only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// A waiting role gives up when the bounded wait runs out or another role has
// already given up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Smem& sm,
                                              const DevCtl& ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*(volatile int*)&sm.abort) return false;
    if ((unsigned long long)(clock64() - t0) > ctl.wait_limit) {
      record_status(ctl, kStatusTimeout);
      *(volatile int*)&sm.abort = 1;
      return false;
    }
  }
  return true;
}

// Ring bookkeeping.  K/V item u (in consumption order) lives in stage
// (u + kQStages) % kStages.  Stages 0..kQStages-1 first hold Q, so their
// first release is "Q moved to TMEM".
__device__ __forceinline__ int item_stage(uint32_t u) { return (int)((u + kQStages) % kStages); }
// releases of the stage that must have happened before item u may be loaded
__device__ __forceinline__ uint32_t item_releases(uint32_t u) { return (u + kQStages) / kStages; }
// earlier fills (by TMA) of item u's stage
__device__ __forceinline__ uint32_t item_fills(uint32_t u) {
  return (u + kQStages) / kStages - (item_stage(u) < kQStages ? 1u : 0u);
}

struct KvTile {
  int src;       // 0: k/v (prefill keys or suffix keys), 1: cached prefix
  int tile;      // tile index within its source
  bool partial;
  bool any_fast;
};

// Key tile number `idx` of this CTA's list.  Suffix mode lists the cache
// tiles first (all visible; the last may be ragged), then the suffix tiles.
template <bool kSuffix>
__device__ __forceinline__ KvTile kv_tile_at(const Smem& sm, int idx, int n_cache, int P) {
  if (kSuffix && idx < n_cache) return KvTile{1, idx, (idx + 1) * kBN > P, false};
  const uint16_t e = sm.list[kSuffix ? idx - n_cache : idx];
  return KvTile{0, (int)(e & kTileIndex), (e & kTilePartial) != 0, (e & kTileAnyFast) != 0};
}

template <bool kSuffix>
__global__ void __launch_bounds__(kThreads, 1)
    tc_attention_kernel(const __grid_constant__ TcParams p, const DevCtl ctl) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Smem& sm = *reinterpret_cast<Smem*>(smem + kOffCtl);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOffCodes);
  uint8_t* ring = smem;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_per_b = p.Sq * p.Hq;
  const int n_qtiles = (rows_per_b + kBM - 1) / kBM;
  const int qtile = blockIdx.x % n_qtiles;
  const int split = blockIdx.x / n_qtiles;
  const int b = blockIdx.y;
  const int row0 = qtile * kBM;
  const int tok_per_tile = kBM / p.Hq;
  const int tq0 = qtile * tok_per_tile;
  const int tq1 = min(tq0 + tok_per_tile, p.Sq) - 1;   // last valid query token
  const int n_key_tok = p.Sq;                           // tokens that carry codes
  const int n_cache = kSuffix ? (p.P + kBN - 1) / kBN : 0;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_tmem, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_q);
    tma_prefetch_desc(&p.map_k);
    tma_prefetch_desc(&p.map_v);
    if (kSuffix) {
      tma_prefetch_desc(&p.map_kc);
      tma_prefetch_desc(&p.map_vc);
    }
    // Q does not depend on the mask: start it before the scan.  One 4-D box
    // brings all four 64-column blocks of the 128-row tile.
    mbar_arrive_expect_tx(&sm.q_full, 4 * kQBlk);
    tma_load_4d(ring, &p.map_q, &sm.q_full, 0, row0, 0, b);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  {
    const uint8_t* ar = p.ar + (long long)b * p.mask_bs;
    const int32_t* seg = (!kSuffix && p.seg) ? p.seg + (long long)b * p.mask_bs : nullptr;
    build_codes_x32<kThreads>(ar, seg, n_key_tok, pad_tokens(n_key_tok), codes, sm.scan);
  }
  // Query-tile summary, then per-key-tile classification.
  if (warp == 0) {
    int any_e = 0, all_e = 1;
    for (int t = tq0 + lane; t <= tq1; t += 32) {
      const int e = (codes[t] >> 1) & 1;
      any_e |= e;
      all_e &= e;
    }
    any_e = __any_sync(0xffffffffu, any_e);
    all_e = __all_sync(0xffffffffu, all_e);
    if (lane == 0) {
      sm.q_any_exp = any_e;
      sm.q_all_exp = all_e;
      sm.cq_first = codes[tq0];
      sm.cq_last = codes[tq1];
    }
  }
  __syncthreads();
  const int n_ktiles = (n_key_tok + kBN - 1) / kBN;
  {
    const uint32_t csq0 = sm.cq_first >> 2, csq1 = sm.cq_last >> 2;
    const int q_any_exp = sm.q_any_exp, q_all_exp = sm.q_all_exp;
    for (int t = warp; t < n_ktiles; t += kThreads / 32) {
      const int k0 = t * kBN;
      const int k1 = min(k0 + kBN, n_key_tok) - 1;
      int any_f = 0, all_f = 1;
      for (int j = k0 + lane; j <= k1; j += 32) {
        const int f = codes[j] & 1;
        any_f |= f;
        all_f &= f;
      }
      any_f = __any_sync(0xffffffffu, any_f);
      all_f = __all_sync(0xffffffffu, all_f);
      if (lane == 0) {
        const uint32_t csk0 = codes[k0] >> 2, csk1 = codes[k1] >> 2;
        uint8_t c;
        if (csk0 > csq1 || (q_all_exp && all_f)) {
          c = 0;  // no query of the tile sees any key of it
        } else if (csk1 <= csq0 && !(q_any_exp && any_f) && k1 - k0 + 1 == kBN) {
          c = 1;  // every query sees every key
        } else {
          c = 2;  // per-row visible prefix (and FAST hole)
        }
        sm.cls[t] = c | (any_f ? 4 : 0);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    for (int t0 = 0; t0 < n_ktiles; t0 += 32) {
      const int t = t0 + lane;
      const uint8_t c = t < n_ktiles ? sm.cls[t] : 0;
      const unsigned m = __ballot_sync(0xffffffffu, (c & 3) != 0);
      if (c & 3) {
        const int pos = base + __popc(m & ((1u << lane) - 1));
        sm.list[pos] = (uint16_t)(t | ((c & 3) == 2 ? kTilePartial : 0) |
                                  ((c & 4) ? kTileAnyFast : 0));
      }
      base += __popc(m);
    }
    if (lane == 0) sm.n_list = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sm.tmem_base;
  const uint32_t tO = tmem + kColO;
  const uint32_t tQ = tmem + kColQ;
  const uint32_t tS = tmem + kColS;      // S[b] at +64*b

  // This CTA's slice of the key-tile list.
  const int n_total = n_cache + sm.n_list;
  const int per = (n_total + p.n_splits - 1) / p.n_splits;
  const int it_begin = min(split * per, n_total);
  const int it_end = min(it_begin + per, n_total);
  const int n_it = it_end - it_begin;

  // The producer and MMA warps walk their schedules with all 32 lanes (a
  // warp-uniform control flow keeps addresses and descriptors in uniform
  // registers); lane 0 alone issues every TMA / MMA / commit.  It must be one
  // FIXED thread: tcgen05.mma ordering and tcgen05.commit tracking are per
  // issuing thread, and MMAs issued from different lanes may overlap (with
  // elect.sync choosing the issuer, PV accumulations into O raced).
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (n_it > 0) {
      uint32_t u = 0;
      auto load = [&](int idx, bool is_v) -> bool {
        const KvTile kt = kv_tile_at<kSuffix>(sm, idx, n_cache, p.P);
        const int s = item_stage(u);
        const uint32_t rel = item_releases(u);
        if (rel > 0) {
          bool ok = wait_or_abort(&sm.kv_empty[s], (rel - 1) & 1, sm, ctl);
          if (!__all_sync(0xffffffffu, ok)) return false;
        }
        const CUtensorMap* map = kt.src ? (is_v ? &p.map_vc : &p.map_kc)
                                        : (is_v ? &p.map_v : &p.map_k);
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.kv_full[s], kItemBytes);
          tma_load_4d(ring + s * kItemBytes, map, &sm.kv_full[s], 0, kt.tile * kBN, 0, b);
        }
        __syncwarp();
        ++u;
        return true;
      };
      bool ok = true;
      for (int i = it_begin; i < it_end && ok; ++i) {
        ok = load(i, false);
        if (ok && i > it_begin) ok = load(i - 1, true);
      }
      if (ok) ok = load(it_end - 1, true);
      if (!ok) {  // drain: every issued load must land before the CTA exits
        for (uint32_t w = (u > kStages ? u - kStages : 0); w < u; ++w)
          (void)mbar_wait(&sm.kv_full[item_stage(w)], item_fills(w) & 1, ctl);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (n_it > 0) {
      bool ok = __all_sync(0xffffffffu, wait_or_abort(&sm.q_tmem, 0, sm, ctl));
      tc_fence_after();
      const uint32_t ring_base = smem_u32(ring);
      // Descriptors are linear in the start address (bits 0-13 = addr >> 4),
      // so a stage's base descriptor plus a constant addresses each K step.
      const uint64_t kdesc0 = sdesc_sw128(ring_base, 16, 1024);     // K: K-major
      const uint64_t vdesc0 = sdesc_sw128(ring_base, kBlk, 1024);   // V: MN-major
      uint32_t u = 0;
      auto pv = [&](int x) -> bool {
        const int bp = x & 1;
        if (!__all_sync(0xffffffffu, wait_or_abort(&sm.p_full[bp], (x >> 1) & 1, sm, ctl)))
          return false;
        const int s = item_stage(u);
        if (!__all_sync(0xffffffffu, wait_or_abort(&sm.kv_full[s], item_fills(u) & 1, sm, ctl)))
          return false;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t vd = vdesc0 + (uint64_t)((s * kItemBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // B = V[16 keys x 256 d], MN-major: 8-key groups 1024 B apart,
            // 64-wide d blocks one block (8 KB) apart; a K step is 16 rows.
            umma_ts(tO, tS + 64 * bp + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), kIdescPV,
                    (x > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&sm.kv_empty[s]);
          umma_commit(&sm.o_done);
        }
        __syncwarp();
        ++u;
        return true;
      };
      for (int i = it_begin; i < it_end && ok; ++i) {
        const int li = i - it_begin;
        const int s = item_stage(u);
        ok = __all_sync(0xffffffffu, wait_or_abort(&sm.kv_full[s], item_fills(u) & 1, sm, ctl));
        if (!ok) break;
        if (li >= 2) {
          // S[li%2] still holds P of tile li-2, the A operand of PV(li-2).
          // MMAs issued by one thread are pipelined, not serialised, so the
          // write of this QK must wait until that PV has finished reading.
          ok = __all_sync(0xffffffffu, wait_or_abort(&sm.o_done, (li - 2) & 1, sm, ctl));
          if (!ok) break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint64_t kd = kdesc0 + (uint64_t)((s * kItemBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            // B = K[64 keys x 16 d], K-major: 8-row groups 1024 B apart; the
            // K step walks 32 B inside a 64-column block, then the next block.
            umma_ts(tS + 64 * (li & 1), tQ + kk * 8,
                    kd + (uint64_t)(((kk >> 2) * kBlk + (kk & 3) * 32) >> 4), kIdescQK,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm.kv_empty[s]);
          umma_commit(&sm.s_full[li & 1]);
        }
        __syncwarp();
        ++u;
        if (li >= 1) ok = pv(li - 1);
      }
      if (ok) ok = pv(n_it - 1);
      // Whatever happened, let every issued MMA finish before TMEM is freed.
      if (lane == 0) umma_commit(&sm.drain);
      __syncwarp();
      (void)mbar_wait(&sm.drain, 0, ctl);
    }
  } else {
    // ---------------------------------------- Q -> TMEM, softmax, epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // tile row of this thread
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int tok = min(tq0 + r / p.Hq, tq1);      // padding rows reuse the last token
    const uint32_t cq = codes[tok];
    const uint32_t csq = cq >> 2;
    const bool row_expert = (cq & 2u) != 0;
    const float c = p.scale_log2;                  // > 0
    float m_run = -INFINITY;  // running max of scaled scores (log2 units)
    float l_run = 0.f;
    bool ok = true;

    if (n_it > 0) {
      // Q rows: smem (TMA, swizzled) -> registers -> TMEM columns [256, 384).
      ok = wait_or_abort(&sm.q_full, 0, sm, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          const uint8_t* rowp = ring + cb * kQBlk + r * 128;
          uint32_t w[32];
#pragma unroll
          for (int u16 = 0; u16 < 8; ++u16) {
            const uint4 v4 = *reinterpret_cast<const uint4*>(rowp + ((u16 ^ (r & 7)) << 4));
            w[4 * u16 + 0] = v4.x;
            w[4 * u16 + 1] = v4.y;
            w[4 * u16 + 2] = v4.z;
            w[4 * u16 + 3] = v4.w;
          }
          tmem_st32(tQ + lane_off + 32 * cb, w);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();  // the ring stages holding Q are refilled by TMA
      tc_fence_before();
      softmax_bar();
      if (warp == 2 && lane == 0) {
        mbar_arrive(&sm.q_tmem);
        for (int s = 0; s < kQStages; ++s) mbar_arrive(&sm.kv_empty[s]);
      }
    }

    for (int i = it_begin; i < it_end && ok; ++i) {
      const int li = i - it_begin;
      const int bs = li & 1;
      if (!wait_or_abort(&sm.s_full[bs], (li >> 1) & 1, sm, ctl)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const KvTile kt = kv_tile_at<kSuffix>(sm, i, n_cache, p.P);
      float x[kBN];
      {
        uint32_t raw0[32], raw1[32];
        tmem_ld32(tS + lane_off + 64 * bs, raw0);
        tmem_ld32(tS + lane_off + 64 * bs + 32, raw1);
        tmem_ld_wait();
        reg_fence(raw0);
        reg_fence(raw1);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          x[e] = __uint_as_float(raw0[e]);
          x[32 + e] = __uint_as_float(raw1[e]);
        }
      }
      if (kt.partial) {
        const int k0 = kt.tile * kBN;
        int e;              // keys [0, e) of the tile pass the cumsum rule
        bool hole = false;  // expert row and the tile holds FAST keys
        if (kSuffix && kt.src == 1) {
          e = min(kBN, p.P - k0);
        } else {
          // codes are sorted by cs: count the keys with cs <= cs(query)
          e = 0;
#pragma unroll
          for (int step = kBN; step >= 1; step >>= 1) {
            const int probe = e + step;
            if (probe <= kBN && (uint32_t)(codes[k0 + probe - 1] >> 2) <= csq) e = probe;
          }
          e = min(e, n_key_tok - k0);
          hole = row_expert && kt.any_fast;
        }
        if (hole) {
          const uint4* kc = reinterpret_cast<const uint4*>(codes + k0);
#pragma unroll
          for (int g = 0; g < kBN / 8; ++g) {
            const uint4 v4 = kc[g];
            const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              const int j = 8 * g + h;
              const bool fast = ((wv[h >> 1] >> (16 * (h & 1))) & 1u) != 0;
              x[j] = (j < e && !fast) ? x[j] : -INFINITY;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < kBN; ++j) x[j] = j < e ? x[j] : -INFINITY;
        }
      }
      // row max: tree of independent fmax
      float mt[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) mt[j] = fmaxf(fmaxf(x[j], x[j + 16]), fmaxf(x[j + 32], x[j + 48]));
#pragma unroll
      for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) mt[j] = fmaxf(mt[j], mt[j + w]);
      const float mx = mt[0] * c;

      // Lazy rescaling: the reference max only moves when the tile's max
      // exceeds it by more than the threshold, so O (in TMEM) is rarely
      // touched.  Exact: O and l always share the same reference.
      const bool upd = mx > m_run + kRescaleThreshold;
      const float m_new = upd ? mx : m_run;
      const float alpha = ex2(m_run - m_new);      // 0 when m_run = -inf
      const bool need_o = upd && (m_run != -INFINITY);
      l_run *= (m_run == -INFINITY) ? 0.f : alpha;
      m_run = m_new;
      if (__any_sync(0xffffffffu, need_o)) {
        // O holds PV of the previous tile: wait for it, then rescale rows.
        if (!wait_or_abort(&sm.o_done, (li - 1) & 1, sm, ctl)) ok = false;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
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
      const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
      uint32_t pk[32];
      float ls[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = ex2(fmaf(x[2 * e], c, nm));
        const float p1 = ex2(fmaf(x[2 * e + 1], c, nm));
        ls[e & 7] += p0 + p1;
        pk[e] = pack_bf16x2(p0, p1);
      }
      tmem_st32(tS + lane_off + 64 * bs, pk);
      l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sm.p_full[bs]);
    }

    if (ok && n_it > 0) {
      if (!wait_or_abort(&sm.o_done, (n_it - 1) & 1, sm, ctl)) ok = false;
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && n_it > 0) {
      tc_fence_after();
      const long long grow = (long long)b * rows_per_b + row0 + r;   // global row
      const bool row_valid = row0 + r < rows_per_b;
      if (p.n_splits == 1) {
        const float inv = 1.f / l_run;
        // The ring is idle once the last PV is done: stage the bf16 rows there.
        uint8_t* stage = ring + quarter * 16384;
#pragma unroll 1
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * cc, o);
          tmem_ld_wait();
          reg_fence(o);
          uint32_t ob[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            ob[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                __uint_as_float(o[2 * e + 1]) * inv);
          uint8_t* blk = stage + (cc >> 1) * 4096 + lane * 128;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int unit = (cc & 1) * 4 + q4;
            *reinterpret_cast<uint4*>(blk + ((unit ^ (lane & 7)) << 4)) =
                make_uint4(ob[4 * q4], ob[4 * q4 + 1], ob[4 * q4 + 2], ob[4 * q4 + 3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(&p.map_o, stage, 0, row0 + quarter * 32, 0, b);
          tma_store_commit();
          tma_store_wait_all();
        }
        if (!kSuffix && p.lse && row_valid)
          p.lse[grow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      } else if (row_valid) {
        // Split-K partial: unnormalised O and (m, l) for the combine kernel.
        const long long slot = ((long long)split * p.B + b) * rows_per_b + row0 + r;
        float* wo = p.ws + slot * kD;
#pragma unroll 1
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * cc, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(wo + 32 * cc + e) =
                make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                            __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
        }
        float* wml = p.ws + (long long)p.n_splits * p.B * rows_per_b * kD + slot * 2;
        wml[0] = m_run;
        wml[1] = l_run;
      }
    }
    if (n_it == 0 && p.n_splits > 1 && row0 + r < rows_per_b) {
      // An empty split contributes nothing: l = 0 and m = -inf.
      const long long slot = ((long long)split * p.B + b) * rows_per_b + row0 + r;
      float* wml = p.ws + (long long)p.n_splits * p.B * rows_per_b * kD + slot * 2;
      wml[0] = -INFINITY;
      wml[1] = 0.f;
    }
  }

  __syncwarp();  // reconverge the single-lane roles before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merges split-K partials: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One warp per output row; each lane handles 8 of the 256 columns.
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ ws, __nv_bfloat16* __restrict__ out, int n_splits,
                   long long n_rows) {
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
  const float inv = 1.f / L;
  uint4 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + row * kD + lane * 8) = pk;
}

size_t smem_bytes(int n_code_tokens) {
  return 1024 /* alignment slack */ + kOffCodes + (size_t)pad_tokens(n_code_tokens) * 2;
}

}  // namespace

int tc_suffix_splits(int B, int Sq, int P, int Hq) {
  (void)B; (void)Sq; (void)P; (void)Hq;
  return 1;
}

size_t tc_suffix_workspace_bytes(int B, int Sq, int P, int Hq) {
  const int s = tc_suffix_splits(B, Sq, P, Hq);
  if (s <= 1) return 0;
  const size_t rows = (size_t)B * Sq * Hq;
  return (size_t)s * rows * (kD + 2) * sizeof(float);
}

cudaError_t launch_tc_attention(const TcParams& p, bool suffix_mode, const DevCtl& ctl,
                                cudaStream_t st) {
  const int rows = p.Sq * p.Hq;
  const int n_qtiles = (rows + kBM - 1) / kBM;
  dim3 grid(n_qtiles * p.n_splits, p.B);
  const size_t smem = smem_bytes(p.Sq);
  // The opt-in shared-memory size is raised once per process to the largest
  // this kernel can ask for, so later launches (and stream captures) make no
  // attribute calls.
  static const cudaError_t attr_err = [] {
    const int most = (int)smem_bytes(kMaxTokens);
    cudaError_t a = cudaFuncSetAttribute(tc_attention_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    cudaError_t b = cudaFuncSetAttribute(tc_attention_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    return a != cudaSuccess ? a : b;
  }();
  if (attr_err != cudaSuccess) return attr_err;
  if (suffix_mode) {
    tc_attention_kernel<true><<<grid, kThreads, smem, st>>>(p, ctl);
  } else {
    tc_attention_kernel<false><<<grid, kThreads, smem, st>>>(p, ctl);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.n_splits <= 1) return e;
  const long long n_rows = (long long)p.B * rows;
  // The combine writes the bf16 output rows directly (same [B, Sq, Hq, 256] layout).
  combine_kernel<<<(unsigned)((n_rows + 7) / 8), 256, 0, st>>>(
      p.ws, reinterpret_cast<__nv_bfloat16*>(p.out_ptr), p.n_splits, n_rows);
  return cudaGetLastError();
}

}  // namespace piattn
