// noalloc.cu -- pi_attn_suffix_noalloc: the suffix pass with its split-K
// scratch in a fixed device buffer owned by the library, for callers that
// cannot allocate device memory.  The method itself has no such call: it is
// plumbing around pi_attn_suffix, which it calls unchanged.
//
// The buffer is a file-scope __device__ array (one copy per device context,
// created with the module).  Its address is looked up on every call with
// cudaGetSymbolAddress (a host-side table lookup), so it stays right after
// the context is reset and the module reloaded; no call here allocates or
// frees memory.
#include "../../include/pi_attn.h"

namespace {

// Split-K partials need (splits x rows x (256 + 2) floats); the split count
// times the CTA count never exceeds the SM count, and 16 MiB covers every
// pi0-sized suffix batch (816-token cache, 51 tokens x 8 heads, B <= 16).
constexpr size_t kStaticWsBytes = size_t(16) << 20;

__device__ __align__(256) unsigned char g_suffix_ws[kStaticWsBytes];

void* static_ws_ptr() {
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_suffix_ws) == cudaSuccess ? p : nullptr;
}

}  // namespace

extern "C" {

size_t pi_attn_suffix_noalloc_capacity(void) { return kStaticWsBytes; }

int pi_attn_suffix_noalloc(const pi_attn_desc* d, const void* q_suf, const void* k_suf,
                           const void* v_suf, const void* k_cache, const void* v_cache,
                           const uint8_t* ar_mask_suf, void* out, pi_stream_t stream) {
  if (!d) return PI_ERR_ARG;
  // Host-only size check first: an oversize request launches nothing.
  if (pi_attn_suffix_workspace_bytes(d) > kStaticWsBytes) return PI_ERR_UNSUPPORTED;
  if (d->B == 0 || d->Sq == 0)   // nothing to do: validation only, as pi_attn_suffix
    return pi_attn_suffix(d, q_suf, k_suf, v_suf, k_cache, v_cache, ar_mask_suf, out, nullptr,
                          0, stream);
  void* ws = static_ws_ptr();
  if (!ws) return PI_ERR_CUDA;
  return pi_attn_suffix(d, q_suf, k_suf, v_suf, k_cache, v_cache, ar_mask_suf, out, ws,
                        kStaticWsBytes, stream);
}

}  // extern "C"
