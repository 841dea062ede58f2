// tc_attention.cu -- bf16 joint (prefix-LM) attention on tcgen05 tensor cores.
//
// One CTA computes one 128-row query tile: 128 / Hq query tokens x Hq heads.
// In the token-major [B, S, Hq, 256] layout those rows are contiguous, and
// with a single KV head they all read the same K/V rows, so every K/V tile
// brought into shared memory serves all heads ("π0.5 vs MM-DiT joint
// attention", "joint attention 只管算子": 8 query heads, 1 KV head, head_dim
// 256, one shared KV pool).
//
// Per KV tile of 128 keys:
//   S  = Q K^T     tcgen05.mma kind::f16, A = Q (smem), B = K (smem), D in TMEM
//   P  = exp2(S * scale*log2e - m)   fp32 online softmax, one thread per row
//   O += P V       tcgen05.mma, A = P (TMEM, bf16), B = V (smem, MN-major)
// The mask is evaluated in-kernel from the packed codes of mask.cuh: KV tiles
// that no query of the tile can see are never loaded; tiles every query sees
// in full skip the per-element predicate.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Q once, then K/V tiles through a 2-stage ring
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..5  softmax, O correction and the epilogue; warp w owns TMEM
//               lanes / tile rows 32*(w%4) .. 32*(w%4)+31
//
// TMEM (512 columns): O fp32 [0,256), S0 [256,384), S1 [384,512); P of tile t
// is written as packed bf16 over the first 64 columns of S[t%2].
//
// Shared memory: Q 64 KB | KV ring 2 x 64 KB | barriers | per-token codes.
// Every operand tile is 4 column blocks of [rows x 64 bf16] with the 128-byte
// swizzle, as TMA writes it and as the UMMA descriptors describe it.
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
constexpr int kBM = 128;               // query rows per tile
constexpr int kBN = 128;               // keys per KV tile
constexpr int kD = 256;                // head dim
constexpr int kChunkBytes = kBN * 128; // one [128 rows x 64 bf16] swizzled block
constexpr int kTileBytes = 4 * kChunkBytes;  // 64 KB: [128 x 256] bf16
constexpr int kStages = 2;
constexpr int kMaxListTiles = 130;     // ceil(16383 / 128) + slack
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 256

constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, kD, false, true);

struct __align__(8) Smem {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_list;       // entries in `list` (prefill: all key tiles; suffix: suffix tiles)
  int q_any_exp, q_all_exp;
  uint32_t cq_first, cq_last;
  int scan[33];
  uint16_t list[kMaxListTiles];   // tile index | 0x8000 if partial
  uint8_t cls[kMaxListTiles];
};

// Offsets inside the 1024-aligned dynamic shared memory block.
constexpr int kOffQ = 0;
constexpr int kOffKV = kTileBytes;
constexpr int kOffCtl = kOffKV + kStages * kTileBytes;
constexpr int kOffCodes = kOffCtl + ((int)sizeof(Smem) + 127) / 128 * 128;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// Key tile number `idx` of this CTA's work list -> (source, tile, partial).
// Prefill: source 0 = k/v.  Suffix: the cache tiles come first (source 1 =
// k_cache/v_cache), then the suffix tiles of `list` (source 0 = k_suf/v_suf).
struct KvTile {
  int src;
  int tile;
  bool partial;
};

template <bool kSuffix>
__device__ __forceinline__ KvTile kv_tile_at(const Smem& sm, int idx, int n_cache, int P) {
  if (kSuffix && idx < n_cache) {
    return KvTile{1, idx, (idx + 1) * kBN > P};
  }
  const int li = kSuffix ? idx - n_cache : idx;
  const uint16_t e = sm.list[li];
  return KvTile{0, (int)(e & 0x7FFF), (e & 0x8000) != 0};
}

template <bool kSuffix>
__global__ void __launch_bounds__(kThreads, 1)
    tc_attention_kernel(const __grid_constant__ TcParams p, const DevCtl ctl) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Smem& sm = *reinterpret_cast<Smem*>(smem + kOffCtl);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOffCodes);
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;

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
  const int n_key_tok = p.Sq;                           // tokens with codes
  const int n_cache = kSuffix ? (p.P + kBN - 1) / kBN : 0;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
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
    // Q does not depend on the mask: start it before the scan.
    mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
    for (int c = 0; c < 4; ++c)
      tma_load_3d(sQ + c * kChunkBytes, &p.map_q, &sm.q_full, c * 64, row0, b);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  {
    const uint8_t* ar = p.ar + (long long)b * p.mask_bs;
    const int32_t* seg = (!kSuffix && p.seg) ? p.seg + (long long)b * p.mask_bs : nullptr;
    build_codes<uint16_t>(ar, seg, n_key_tok, codes, sm.scan);
  }
  // Query-tile summary and per-key-tile classification.
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
      const uint32_t csq0 = sm.cq_first >> 2, csq1 = sm.cq_last >> 2;
      const uint32_t csk0 = codes[k0] >> 2, csk1 = codes[k1] >> 2;
      uint8_t c;
      if (csk0 > csq1 || (sm.q_all_exp && all_f)) {
        c = 0;  // no query of the tile sees any key of it
      } else if (csk1 <= csq0 && !(sm.q_any_exp && any_f) && k1 - k0 + 1 == kBN) {
        c = 1;  // every query sees every key
      } else {
        c = 2;  // per-element predicate
      }
      sm.cls[t] = c;
    }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    for (int t0 = 0; t0 < n_ktiles; t0 += 32) {
      const int t = t0 + lane;
      const uint8_t c = t < n_ktiles ? sm.cls[t] : 0;
      const unsigned m = __ballot_sync(0xffffffffu, c != 0);
      if (c != 0) {
        const int pos = base + __popc(m & ((1u << lane) - 1));
        sm.list[pos] = (uint16_t)(t | (c == 2 ? 0x8000 : 0));
      }
      base += __popc(m);
    }
    if (lane == 0) sm.n_list = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sm.tmem_base;
  const uint32_t tO = tmem;          // columns [0, 256)
  const uint32_t tS = tmem + 256;    // S[b] at +128*b

  // This CTA's slice of the key-tile list.
  const int n_total = n_cache + sm.n_list;
  const int per = (n_total + p.n_splits - 1) / p.n_splits;
  const int it_begin = min(split * per, n_total);
  const int it_end = min(it_begin + per, n_total);
  const int n_it = it_end - it_begin;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_it > 0) {
      uint32_t u = 0;
      auto load = [&](int idx, bool is_v) -> bool {
        const KvTile kt = kv_tile_at<kSuffix>(sm, idx, n_cache, p.P);
        const int s = u & 1;
        if (!wait_or_abort(&sm.kv_empty[s], ((u >> 1) & 1) ^ 1, sm, ctl)) return false;
        const CUtensorMap* map = kt.src ? (is_v ? &p.map_vc : &p.map_kc)
                                        : (is_v ? &p.map_v : &p.map_k);
        uint8_t* dst = sKV + s * kTileBytes;
        mbar_arrive_expect_tx(&sm.kv_full[s], kTileBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(dst + c * kChunkBytes, map, &sm.kv_full[s], c * 64, kt.tile * kBN, b);
        ++u;
        return true;
      };
      bool ok = true;
      for (int i = it_begin; i < it_end && ok; ++i) {
        ok = load(i, false);
        if (ok && i > it_begin) ok = load(i - 1, true);
      }
      if (ok) ok = load(it_end - 1, true);
      // Drain: every issued load must land before the CTA may exit.
      if (!ok) {
        for (uint32_t w = (u >= 2 ? u - 2 : 0); w < u; ++w)
          (void)mbar_wait(&sm.kv_full[w & 1], (w >> 1) & 1, ctl);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n_it > 0) {
      bool ok = wait_or_abort(&sm.q_full, 0, sm, ctl);
      tc_fence_after();
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      uint32_t u = 0;
      auto pv = [&](int x) -> bool {
        const int bp = x & 1;
        if (!wait_or_abort(&sm.p_full[bp], (x >> 1) & 1, sm, ctl)) return false;
        const int s = u & 1;
        if (!wait_or_abort(&sm.kv_full[s], (u >> 1) & 1, sm, ctl)) return false;
        tc_fence_after();
        const uint32_t v_base = kv_base + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // B = V[16 keys x 256 d], MN-major: 8-key groups 1024 B apart,
          // 64-wide d blocks one chunk apart.
          const uint64_t bdesc = sdesc_sw128(v_base + kk * 2048, kChunkBytes, 1024);
          umma_ts(tO, tS + 128 * bp + kk * 8, bdesc, kIdescPV, (x > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&sm.kv_empty[s]);
        umma_commit(&sm.o_done);
        ++u;
        return true;
      };
      for (int i = it_begin; i < it_end && ok; ++i) {
        const int li = i - it_begin;
        const int s = u & 1;
        if (!(ok = wait_or_abort(&sm.kv_full[s], (u >> 1) & 1, sm, ctl))) break;
        tc_fence_after();
        const uint32_t k_base = kv_base + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          const uint64_t adesc = sdesc_sw128(q_base + off, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(k_base + off, 16, 1024);
          umma_ss(tS + 128 * (li & 1), adesc, bdesc, kIdescQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.kv_empty[s]);
        umma_commit(&sm.s_full[li & 1]);
        ++u;
        if (li >= 1) ok = pv(li - 1);
      }
      if (ok) ok = pv(n_it - 1);
      // Whatever happened, let every issued MMA finish before TMEM is freed.
      umma_commit(&sm.drain);
      (void)mbar_wait(&sm.drain, 0, ctl);
    }
  } else {
    // ------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // tile row of this thread
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int tok = min(tq0 + r / p.Hq, tq1);      // padding rows reuse the last token
    const uint32_t cq = codes[tok];
    float m_run = -INFINITY;  // running max of scaled scores (log2 units)
    float l_run = 0.f;
    bool ok = true;

    for (int i = it_begin; i < it_end; ++i) {
      const int li = i - it_begin;
      const int bs = li & 1;
      if (!wait_or_abort(&sm.s_full[bs], (li >> 1) & 1, sm, ctl)) { ok = false; }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const KvTile kt = kv_tile_at<kSuffix>(sm, i, n_cache, p.P);
      float x[kBN];
      {
        uint32_t raw[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tS + lane_off + 128 * bs + 32 * c, raw);
          tmem_ld_wait();
          reg_fence(raw);
#pragma unroll
          for (int e = 0; e < 32; ++e) x[32 * c + e] = __uint_as_float(raw[e]) * p.scale_log2;
        }
      }
      if (kt.partial) {
        const int k0 = kt.tile * kBN;
        if (kSuffix && kt.src == 1) {
#pragma unroll
          for (int j = 0; j < kBN; ++j)
            if (k0 + j >= p.P) x[j] = -INFINITY;
        } else {
#pragma unroll
          for (int j = 0; j < kBN; ++j) {
            const int kj = k0 + j;
            const bool vis = kj < n_key_tok && visible(cq, codes[min(kj, n_key_tok - 1)]);
            if (!vis) x[j] = -INFINITY;
          }
        }
      }
      float mx = x[0];
#pragma unroll
      for (int j = 1; j < kBN; ++j) mx = fmaxf(mx, x[j]);

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
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * c, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
          tmem_st32(tO + lane_off + 32 * c, o);
        }
      }
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(x[32 * c + 2 * e] - mref);
          const float p1 = ex2(x[32 * c + 2 * e + 1] - mref);
          lsum += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + lane_off + 128 * bs + 16 * c, pk);
      }
      l_run += lsum;
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
        uint8_t* stage = sQ + quarter * 16384;  // Q is dead once the last PV is done
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * c, o);
          tmem_ld_wait();
          reg_fence(o);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                __uint_as_float(o[2 * e + 1]) * inv);
          uint8_t* blk = stage + (c >> 1) * 4096 + lane * 128;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int unit = (c & 1) * 4 + q4;
            *reinterpret_cast<uint4*>(blk + ((unit ^ (lane & 7)) << 4)) =
                make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int c = 0; c < 4; ++c)
            tma_store_3d(&p.map_o, stage + c * 4096, c * 64, row0 + quarter * 32, b);
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
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * c, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(wo + 32 * c + e) =
                make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                            __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
        }
        float* wml = p.ws + (long long)p.n_splits * p.B * rows_per_b * kD + slot * 2;
        wml[0] = m_run;
        wml[1] = l_run;
      } else {
        // padding rows of the last tile: nothing to write
      }
    } else if (!ok) {
      // nothing: the status word already holds the timeout
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
  return 1024 /* alignment slack */ + kOffCodes + ((size_t)n_code_tokens * 2 + 15) / 16 * 16;
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
      p.ws, reinterpret_cast<__nv_bfloat16*>(const_cast<void*>(p.out_ptr)), p.n_splits, n_rows);
  return cudaGetLastError();
}

}  // namespace piattn
