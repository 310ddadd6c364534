// kvq_noalloc.cu - decode attention without a caller-provided workspace.
//
// kvq_decode_attn needs a device workspace for its split-K partial results, which the
// caller allocates.  Some callers cannot: code that runs as a plugin of a host runtime
// that owns every byte of device memory and hands out no allocator, or a serving loop
// that must not allocate (and so must not risk a stall or a failed allocation) once it is
// running.  kvq_decode_attn_noalloc runs the same decode kernel with its partials in a
// fixed, library-owned device array instead, so the caller passes only inputs and outputs.
//
// The array lives in this file as a static __device__ variable; every GPU that loads the
// library holds it (KVQ_NOALLOC_SCRATCH_BYTES) until the process exits.  Host code may not
// use the variable's name as an address, so every call looks the device address up, with
// the cache's device current (it checks that first), and passes it to the kernel.  Looking
// it up each time (cheap once the module is loaded) also stays right after a device reset,
// when the module is loaded again at another address.
#include <cuda_runtime.h>

#include <vector>

#include "kvq_internal.h"

using namespace kvq;

namespace {

constexpr size_t kScratchBytes = KVQ_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// Device address of g_decode_scratch on the current device.
int scratch_for_current_device(void **ptr) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return KVQ_E_CUDA;
  *ptr = p;
  return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attn_noalloc(kvq_cache *c, int32_t layer, int32_t n_seqs, const int32_t *seq_ids,
                                       int32_t n_q_heads, const float *q, float softmax_scale, float *out,
                                       kvq_stream_t stream) {
  if (!c || layer < 0 || layer >= c->p.n_layers || n_seqs < 0) return KVQ_E_INVAL;
  if (n_seqs == 0) return KVQ_OK;
  if (!seq_ids || !q || !out || n_q_heads < 1) return KVQ_E_INVAL;
  if (n_q_heads % c->p.n_kv_heads) return KVQ_E_INVAL;
  if (n_q_heads / c->p.n_kv_heads > MAX_G) return KVQ_E_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u)) return KVQ_E_ALIGN;
  const size_t need = decode_workspace_bytes(c, n_seqs, n_q_heads);
  if (need > kScratchBytes) return KVQ_E_SIZE;
  std::vector<char> seen(c->p.n_seqs, 0);
  std::vector<DecodeSeq> seqs;
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    if (s < 0 || s >= c->p.n_seqs || seen[s]) return KVQ_E_INVAL;
    seen[s] = 1;
    const int64_t n = c->len[(size_t)layer * c->p.n_seqs + s];
    seqs.push_back({s, i, n, quantized_len(c, n)});
  }
  // the scratch array of the cache's own device: the call is rejected when another is current
  int rc = check_device(c);
  if (rc) return rc;
  void *scratch = nullptr;
  rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)D);
  return launch_decode(c, layer, seqs, n_q_heads, q, scale, out, scratch, kScratchBytes,
                       reinterpret_cast<cudaStream_t>(stream));
}
