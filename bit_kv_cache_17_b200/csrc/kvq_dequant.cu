// kvq_dequant.cu - reads tokens back out of the cache as fp32.
//
// Quantized token value (rotated basis): ((code * d) * t) * c for kvarn, code * d for qb_0,
// code * d + m for qb_1 (fp32, this order).  Original basis for kvarn: the same fp32
// butterfly as the append rotation (H is its own inverse up to the factor 128, and
// kappa^2 * 128 ~= 1), applied across the warp.  Tail tokens are returned exactly.
#include <cuda_runtime.h>

#include "kvq_codes.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr unsigned FULL = 0xffffffffu;

// One warp per (token, head); lane holds channels 4*lane .. 4*lane+3.
template <int FAM, int BITS>
__global__ void __launch_bounds__(256)
    k_dequant(LayerView L, int seq, int which, int64_t t0, int64_t t1, int64_t Q, int basis, float *out) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t ntok = t1 - t0;
  if (item >= ntok * L.hkv) return;
  const int64_t p = t0 + item / L.hkv;
  const int head = (int)(item % L.hkv);
  float v[4];
  if (FAM == FAM_BF16 || p >= Q) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(ring_row(L, seq, head, which, p) + 4 * lane);
    const float2 a = ring2f(raw.x, L.tail_f16), b = ring2f(raw.y, L.tail_f16);
    v[0] = a.x;
    v[1] = a.y;
    v[2] = b.x;
    v[3] = b.y;
  } else {
    if constexpr (FAM != FAM_BF16) {
      const SubLayout lay = sub_layout(FAM, BITS);
      const uint8_t *sub = subpage_ptr(L, seq, p / GROUP, head, which);
      const int tip = (int)(p % GROUP);
      const __half *dh = reinterpret_cast<const __half *>(sub + lay.d);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ch = 4 * lane + e, blk = ch >> 5;
        const uint32_t f = which == 0 ? k_field<BITS>(sub + tip * 16 * BITS, ch)
                                      : v_field<BITS>(sub + (tip >> 2) * 64 * BITS, tip & 3, ch);
        float x = __fmul_rn((float)code_value<FAM, BITS>(f), __half2float(dh[tip * 4 + blk]));
        if (FAM == FAM_ASYM) x = __fadd_rn(x, __half2float(reinterpret_cast<const __half *>(sub + lay.m)[tip * 4 + blk]));
        if (FAM == FAM_KVARN) {
          x = __fmul_rn(x, __half2float(reinterpret_cast<const __half *>(sub + lay.t)[tip]));
          x = __fmul_rn(x, __half2float(reinterpret_cast<const __half *>(sub + lay.c)[ch]));
        }
        v[e] = x;
      }
      if (FAM == FAM_KVARN && basis == 0) {
        // stages h = 1, 2 inside the lane, h = 4..64 across lanes (xor 1..16)
        float a = v[0], b = v[1];
        v[0] = __fadd_rn(a, b);
        v[1] = __fsub_rn(a, b);
        a = v[2];
        b = v[3];
        v[2] = __fadd_rn(a, b);
        v[3] = __fsub_rn(a, b);
        a = v[0];
        b = v[2];
        v[0] = __fadd_rn(a, b);
        v[2] = __fsub_rn(a, b);
        a = v[1];
        b = v[3];
        v[1] = __fadd_rn(a, b);
        v[3] = __fsub_rn(a, b);
#pragma unroll
        for (int o = 1; o <= 16; o <<= 1) {
          const bool hi = lane & o;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float other = __shfl_xor_sync(FULL, v[e], o);
            v[e] = hi ? __fsub_rn(other, v[e]) : __fadd_rn(v[e], other);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = __fmul_rn(v[e], kKappa());
      }
    }
  }
  float4 *dst = reinterpret_cast<float4 *>(out + ((p - t0) * L.hkv + head) * D + 4 * lane);
  *dst = make_float4(v[0], v[1], v[2], v[3]);
}

}  // namespace

int launch_dequant(const kvq_cache *c, int layer, int seq, int which, int64_t t0, int64_t t1, int basis,
                   float *out, cudaStream_t st) {
  const LayerView L = layer_view(c, layer);
  const int fam = which ? c->fam_v : c->fam_k, bits = which ? c->bits_v : c->bits_k;
  const int64_t n = c->len[(size_t)layer * c->p.n_seqs + seq];
  const int64_t Q = quantized_len(c, n);
  const int64_t items = (t1 - t0) * c->p.n_kv_heads;
  const unsigned grid = (unsigned)((items + 7) / 8);
#define KVQ_DQ(F, B) \
  if (fam == F && bits == B) { k_dequant<F, B><<<grid, 256, 0, st>>>(L, seq, which, t0, t1, Q, basis, out); \
    note_launches(1); return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_E_CUDA; }
  KVQ_DQ(FAM_BF16, 16)
  KVQ_DQ(FAM_SYM, 2) KVQ_DQ(FAM_SYM, 3) KVQ_DQ(FAM_SYM, 4) KVQ_DQ(FAM_SYM, 5) KVQ_DQ(FAM_SYM, 6) KVQ_DQ(FAM_SYM, 8)
  KVQ_DQ(FAM_ASYM, 2) KVQ_DQ(FAM_ASYM, 3) KVQ_DQ(FAM_ASYM, 4) KVQ_DQ(FAM_ASYM, 5) KVQ_DQ(FAM_ASYM, 6)
  KVQ_DQ(FAM_KVARN, 2) KVQ_DQ(FAM_KVARN, 3) KVQ_DQ(FAM_KVARN, 4) KVQ_DQ(FAM_KVARN, 5) KVQ_DQ(FAM_KVARN, 6)
  KVQ_DQ(FAM_KVARN, 8)
#undef KVQ_DQ
  return KVQ_E_UNSUPPORTED;
}

}  // namespace kvq
