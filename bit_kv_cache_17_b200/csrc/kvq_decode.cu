// kvq_decode.cu - split-K decode attention over [quantized prefix | BF16 tail].
//
// Pages: "Fork of beellama and kvarn KV quants at long context" (ai-manual.ru), the
// decode discussion: at long context depth decode is memory bound and the dequantization
// inside attention decides the speed; "KV Cache Precision Tail" of the BeeLLama.cpp
// v0.4.0 page: the newest tokens are read exactly from BF16.
//
// Per (sequence, KV head) the context is cut into splits; one CTA per split computes the
// online-softmax state (m, l, acc) of its G query heads, the last CTA to finish (an atomic
// ticket, no waiting) merges the splits.  For kvarn K the query is rotated once
// (q' = H.q.kappa) and scaled per 256-token page by the channel scales c, so the keys are
// never rotated back; for kvarn V the accumulator stays in the rotated basis and the
// inverse rotation is applied once per head in the merge.
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>

#include "kvq_codes.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int DT = 128;      // threads per CTA
constexpr int NW = DT / 32;  // warps per CTA
constexpr int CH = 32;       // tokens per chunk (one per lane)
constexpr int MAXSQ = 48;    // max splits over the quantized prefix per (seq, head)
constexpr int MAXST = 16;    // max splits over the tail per (seq, head)
constexpr int MAXSPL = MAXSQ + MAXST;
constexpr int PSTRIDE = 2 + D;  // floats per partial: m, l, acc[128]
constexpr int MAXS = 64;        // sequences per launch
constexpr float LOG2E = 1.4426950408889634f;

struct DSeq {
  int32_t seq, row;     // cache slot; row of q / out
  int32_t nsq, nst;     // splits per head over the quantized prefix / the tail
  int32_t cps_q, cps_t; // chunks per split
  int32_t cta0;         // first CTA of this sequence
  int32_t part0;        // first partial slot of this sequence
  int64_t n, Q;
};

struct DArgs {
  int32_t nseq, G, hkv, rotk, rotv, ncta;
  float qscale;  // softmax scale * log2(e)
  const float *q;
  float *out;
  float *ws;
  uint32_t *tickets;
  DSeq s[MAXS];
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

// field of channel ch of a K token held as 32-bit words (indices resolve at compile time)
template <int BITS>
__device__ __forceinline__ uint32_t k_field_w(const uint32_t *w, int ch) {
  constexpr int WL = plane_lo(BITS), WH = plane_hi(BITS);
  const int blk = ch >> 5, e = ch & 31, jj = e >> 2, k = e & 3;
  constexpr int FL = 8 / WL;
  const int bl = 16 * (jj / FL) + 4 * blk + k;
  uint32_t f = (w[bl >> 2] >> (8 * (bl & 3) + (jj % FL) * WL)) & ((1u << WL) - 1u);
  if constexpr (WH > 0) {
    constexpr int FH = 8 / WH;
    const int bh = 16 * WL + 16 * (jj / FH) + 4 * blk + k;
    f |= ((w[bh >> 2] >> (8 * (bh & 3) + (jj % FH) * WH)) & ((1u << WH) - 1u)) << WL;
  }
  return f;
}

template <int FAM, int BITS>
__global__ void __launch_bounds__(DT) k_decode(LayerView L, DArgs A) {
  __shared__ float qraw[MAX_G][D];
  __shared__ float qrot[MAX_G][D];
  __shared__ float qc[NW][MAX_G][D];
  __shared__ float ps[NW][MAX_G][CH];
  __shared__ float qsum[MAX_G][4];
  __shared__ float mw[NW][MAX_G], lw[NW][MAX_G];
  __shared__ float accw[NW][MAX_G][D];
  __shared__ int is_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bid = blockIdx.x;
  int si = 0;
  while (si + 1 < A.nseq && A.s[si + 1].cta0 <= bid) ++si;
  const DSeq &s = A.s[si];
  const int nspl = s.nsq + s.nst;
  const int local = bid - s.cta0;
  const int head = local / nspl, sp = local % nspl;
  const int G = A.G;
  const bool tail = sp >= s.nsq;
  int64_t a, b;
  if (!tail) {
    a = (int64_t)sp * s.cps_q * CH;
    b = min(a + (int64_t)s.cps_q * CH, s.Q);
  } else {
    a = s.Q + (int64_t)(sp - s.nsq) * s.cps_t * CH;
    b = min(a + (int64_t)s.cps_t * CH, s.n);
  }

  // query rows of this KV head, pre-scaled by softmax_scale * log2(e)
  for (int idx = tid; idx < G * D; idx += DT) {
    const int g = idx / D, j = idx % D;
    qraw[g][j] = A.q[((int64_t)s.row * A.hkv * G + head * G + g) * D + j] * A.qscale;
  }
  __syncthreads();
  if (!tail && A.rotk) {
    // q' = H.q.kappa with the same butterfly as the keys' rotation
    if (tid < G) {
      float r[D];
#pragma unroll
      for (int j = 0; j < D; ++j) r[j] = qraw[tid][j];
#pragma unroll
      for (int h = 1; h < D; h <<= 1) {
#pragma unroll
        for (int j = 0; j < D; ++j) {
          if (j & h) continue;
          const float x = r[j], y = r[j + h];
          r[j] = x + y;
          r[j + h] = x - y;
        }
      }
#pragma unroll
      for (int j = 0; j < D; ++j) qrot[tid][j] = r[j] * kKappa();
    }
  } else {
    for (int idx = tid; idx < G * D; idx += DT) qrot[idx / D][idx % D] = qraw[idx / D][idx % D];
  }
  __syncthreads();
  if (FAM == FAM_ASYM && tid < G * 4) {
    const int g = tid / 4, bb = tid % 4;
    float sum = 0.f;
    for (int e = 0; e < 32; ++e) sum += qrot[g][32 * bb + e];
    qsum[g][bb] = sum;
  }
  __syncthreads();

  float m[MAX_G], l[MAX_G], acc[MAX_G][4];
#pragma unroll
  for (int g = 0; g < MAX_G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) acc[g][bb] = 0.f;
  }

  const int64_t nch = (b - a + CH - 1) / CH;
  int64_t cur_page = -1;
  float cv[4] = {1.f, 1.f, 1.f, 1.f};  // V channel scales of the current page (kvarn)
  for (int64_t ci = warp; ci < nch; ci += NW) {
    const int64_t i0 = a + ci * CH;
    const int64_t i = i0 + lane;
    const bool valid = i < b;
    float sc[MAX_G];
#pragma unroll
    for (int g = 0; g < MAX_G; ++g) sc[g] = 0.f;
    const uint8_t *sk = nullptr, *sv = nullptr;
    const SubLayout lay = sub_layout(FAM, BITS);
    if constexpr (FAM != FAM_BF16) {
      if (!tail) {
        const int64_t page = i0 / GROUP;
        sk = subpage_ptr(L, s.seq, page, head, 0);
        sv = subpage_ptr(L, s.seq, page, head, 1);
        const float *qq = &qrot[0][0];
        if (FAM == FAM_KVARN) {
          if (page != cur_page) {
            const __half *ck = reinterpret_cast<const __half *>(sk + lay.c);
            const __half *cvh = reinterpret_cast<const __half *>(sv + lay.c);
            for (int idx = lane; idx < G * D; idx += 32)
              qc[warp][idx / D][idx % D] = qrot[idx / D][idx % D] * __half2float(ck[idx % D]);
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) cv[bb] = __half2float(cvh[lane + 32 * bb]);
            __syncwarp();
            cur_page = page;
          }
          qq = &qc[warp][0][0];
        }
        if (valid) {
          const int tip = (int)(i % GROUP);
          uint32_t w[4 * BITS];
          const uint4 *src = reinterpret_cast<const uint4 *>(sk + tip * 16 * BITS);
#pragma unroll
          for (int k = 0; k < BITS; ++k) reinterpret_cast<uint4 *>(w)[k] = src[k];
          const __half *dk = reinterpret_cast<const __half *>(sk + lay.d);
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {
            float ab[MAX_G];
#pragma unroll
            for (int g = 0; g < MAX_G; ++g) ab[g] = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int ch = 32 * blk + e;
              const float cval = (float)code_value<FAM, BITS>(k_field_w<BITS>(w, ch));
#pragma unroll
              for (int g = 0; g < MAX_G; ++g)
                if (g < G) ab[g] = fmaf(cval, qq[g * D + ch], ab[g]);
            }
            const float d = __half2float(dk[tip * 4 + blk]);
            float mk = 0.f;
            if (FAM == FAM_ASYM) mk = __half2float(reinterpret_cast<const __half *>(sk + lay.m)[tip * 4 + blk]);
#pragma unroll
            for (int g = 0; g < MAX_G; ++g) {
              sc[g] = fmaf(d, ab[g], sc[g]);
              if (FAM == FAM_ASYM) sc[g] = fmaf(mk, qsum[g][blk], sc[g]);
            }
          }
          if (FAM == FAM_KVARN) {
            const float t = __half2float(reinterpret_cast<const __half *>(sk + lay.t)[tip]);
#pragma unroll
            for (int g = 0; g < MAX_G; ++g) sc[g] *= t;
          }
        }
      }
    }
    if (tail && valid) {
      const __nv_bfloat16 *row = ring_row(L, s.seq, head, 0, i);
      for (int j = 0; j < D; j += 8) {
        uint4 raw = *reinterpret_cast<const uint4 *>(row + j);
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float x0 = __low2float(h2[u]), x1 = __high2float(h2[u]);
#pragma unroll
          for (int g = 0; g < MAX_G; ++g)
            if (g < G) sc[g] = fmaf(x1, qraw[g][j + 2 * u + 1], fmaf(x0, qraw[g][j + 2 * u], sc[g]));
        }
      }
    }
    // online softmax over the chunk
#pragma unroll
    for (int g = 0; g < MAX_G; ++g) {
      if (g >= G) break;
      const float sv_ = valid ? sc[g] : -INFINITY;
      const float cm = warp_max(sv_);
      const float mn = fmaxf(m[g], cm);
      const float alpha = m[g] == -INFINITY ? 0.f : exp2f(m[g] - mn);
      const float p = valid ? exp2f(sv_ - mn) : 0.f;
      l[g] = l[g] * alpha + warp_sum(p);
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) acc[g][bb] *= alpha;
      m[g] = mn;
      ps[warp][g][lane] = p;
    }
    __syncwarp();
    const int cnt = (int)((b - i0) < CH ? (b - i0) : CH);
    for (int t = 0; t < cnt; ++t) {
      const int64_t it = i0 + t;
      float vv[4];
      if (tail || FAM == FAM_BF16) {
        const __nv_bfloat16 *row = ring_row(L, s.seq, head, 1, it);
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) vv[bb] = __bfloat162float(row[lane + 32 * bb]);
      } else {
        if constexpr (FAM != FAM_BF16) {
          const SubLayout lv = sub_layout(FAM, BITS);
          const int tip = (int)(it % GROUP);
          const uint8_t *quad = sv + (tip >> 2) * 64 * BITS;
          const __half *dv = reinterpret_cast<const __half *>(sv + lv.d);
          float tv = 1.f;
          if (FAM == FAM_KVARN) tv = __half2float(reinterpret_cast<const __half *>(sv + lv.t)[tip]);
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            const int ch = lane + 32 * bb;
            float val = (float)code_value<FAM, BITS>(v_field<BITS>(quad, tip & 3, ch)) *
                        __half2float(dv[tip * 4 + bb]);
            if (FAM == FAM_ASYM) val += __half2float(reinterpret_cast<const __half *>(sv + lv.m)[tip * 4 + bb]);
            if (FAM == FAM_KVARN) val *= tv * cv[bb];
            vv[bb] = val;
          }
        }
      }
#pragma unroll
      for (int g = 0; g < MAX_G; ++g) {
        if (g >= G) break;
        const float p = ps[warp][g][t];
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acc[g][bb] = fmaf(p, vv[bb], acc[g][bb]);
      }
    }
    __syncwarp();
  }

  // combine the warps of this CTA
#pragma unroll
  for (int g = 0; g < MAX_G; ++g) {
    if (g >= G) break;
    if (lane == 0) {
      mw[warp][g] = m[g];
      lw[warp][g] = l[g];
    }
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) accw[warp][g][lane + 32 * bb] = acc[g][bb];
  }
  __syncthreads();
  const int slot0 = s.part0 + head * nspl;
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mw[w][g]);
    float av = 0.f, lv = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < NW; ++w) {
        if (mw[w][g] == -INFINITY) continue;
        const float f = exp2f(mw[w][g] - M);
        av += f * accw[w][g][tid];
        lv += f * lw[w][g];
      }
    }
    float *dst = A.ws + ((int64_t)(slot0 + sp) * G + g) * PSTRIDE;
    dst[2 + tid] = av;
    if (tid == 0) {
      dst[0] = M;
      dst[1] = lv;
    }
  }

  // the last CTA of this (sequence, KV head) merges all splits
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(&A.tickets[s.seq * A.hkv + head], 1u);
    is_last = prev == (unsigned)(nspl - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  float *buf = &accw[0][0][0];
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
    for (int k = 0; k < nspl; ++k) M = fmaxf(M, __ldcg(A.ws + ((int64_t)(slot0 + k) * G + g) * PSTRIDE));
    float Ls = 0.f, ar = 0.f, ap = 0.f;
    if (M != -INFINITY) {
      for (int k = 0; k < nspl; ++k) {
        const float *src = A.ws + ((int64_t)(slot0 + k) * G + g) * PSTRIDE;
        const float mk = __ldcg(src);
        if (mk == -INFINITY) continue;
        const float f = exp2f(mk - M);
        Ls += f * __ldcg(src + 1);
        const float v = f * __ldcg(src + 2 + tid);
        if (k < s.nsq) ar += v;
        else ap += v;
      }
    }
    if (A.rotv) {
      buf[tid] = ar;
      __syncthreads();
      for (int h = 1; h < D; h <<= 1) {
        const bool lo = !(tid & h);
        float x = 0.f, y = 0.f;
        if (lo) {
          x = buf[tid];
          y = buf[tid + h];
        }
        __syncthreads();
        if (lo) {
          buf[tid] = x + y;
          buf[tid + h] = x - y;
        }
        __syncthreads();
      }
      ar = buf[tid] * kKappa();
      __syncthreads();
    }
    A.out[((int64_t)s.row * A.hkv * G + head * G + g) * D + tid] = Ls > 0.f ? (ar + ap) / Ls : 0.f;
  }
  if (tid == 0) A.tickets[s.seq * A.hkv + head] = 0u;
}

template <int FAM, int BITS>
cudaError_t run(const LayerView &L, const DArgs &A, cudaStream_t st) {
  k_decode<FAM, BITS><<<A.ncta, DT, 0, st>>>(L, A);
  return cudaGetLastError();
}

cudaError_t dispatch(int fam, int bits, const LayerView &L, const DArgs &A, cudaStream_t st) {
#define KVQ_D(F, B) \
  if (fam == F && bits == B) return run<F, B>(L, A, st);
  KVQ_D(FAM_BF16, 16)
  KVQ_D(FAM_SYM, 2) KVQ_D(FAM_SYM, 3) KVQ_D(FAM_SYM, 4) KVQ_D(FAM_SYM, 5) KVQ_D(FAM_SYM, 6) KVQ_D(FAM_SYM, 8)
  KVQ_D(FAM_ASYM, 2) KVQ_D(FAM_ASYM, 3) KVQ_D(FAM_ASYM, 4) KVQ_D(FAM_ASYM, 5) KVQ_D(FAM_ASYM, 6)
  KVQ_D(FAM_KVARN, 2) KVQ_D(FAM_KVARN, 3) KVQ_D(FAM_KVARN, 4) KVQ_D(FAM_KVARN, 5) KVQ_D(FAM_KVARN, 6)
  KVQ_D(FAM_KVARN, 8)
#undef KVQ_D
  return cudaErrorInvalidValue;
}

}  // namespace

size_t decode_workspace_bytes(const kvq_cache *c, int n_seqs, int n_q_heads) {
  const int G = n_q_heads / c->p.n_kv_heads;
  return sizeof(float) * (size_t)std::max(n_seqs, 1) * c->p.n_kv_heads * MAXSPL * G * PSTRIDE;
}

int launch_decode(const kvq_cache *c, int layer, const std::vector<DecodeSeq> &seqs, int n_q_heads,
                  const float *q, float scale, float *out, void *ws, size_t ws_bytes, cudaStream_t st) {
  if (c->p.type_k != c->p.type_v) return KVQ_E_UNSUPPORTED;
  const LayerView L = layer_view(c, layer);
  const int hkv = c->p.n_kv_heads, G = n_q_heads / hkv;
  const double tb = (double)token_bytes(c->fam_k, c->bits_k) + token_bytes(c->fam_v, c->bits_v);
  double total = 0.0;
  for (const DecodeSeq &d : seqs) total += hkv * ((double)d.Q * tb + (double)(d.n - d.Q) * 4.0 * D);
  const double target = 4.0 * c->num_sms;
  (void)ws_bytes;
  for (size_t base = 0; base < seqs.size(); base += MAXS) {
    const size_t cnt = std::min<size_t>(MAXS, seqs.size() - base);
    DArgs A{};
    A.nseq = (int)cnt;
    A.G = G;
    A.hkv = hkv;
    A.rotk = c->fam_k == FAM_KVARN;
    A.rotv = c->fam_v == FAM_KVARN;
    A.qscale = scale * LOG2E;
    A.q = q;
    A.out = out;
    A.ws = static_cast<float *>(ws);
    A.tickets = reinterpret_cast<uint32_t *>(c->base + c->off_tickets);
    int cta = 0, part = 0;
    for (size_t i = 0; i < cnt; ++i) {
      const DecodeSeq &d = seqs[base + i];
      DSeq &s = A.s[i];
      s.seq = d.seq;
      s.row = d.row;
      s.n = d.n;
      s.Q = d.Q;
      const int64_t nchq = (d.Q + CH - 1) / CH, ncht = (d.n - d.Q + CH - 1) / CH;
      auto want = [&](double bytes, int64_t nchunks, int cap) -> int {
        if (nchunks <= 0) return 0;
        int w = total > 0 ? (int)std::ceil(target * hkv * bytes / total / hkv) : 1;
        w = std::max(1, std::min<int>(w, cap));
        return (int)std::min<int64_t>(w, nchunks);
      };
      int wq = want((double)d.Q * tb, nchq, MAXSQ);
      int wt = want((double)(d.n - d.Q) * 4.0 * D, ncht, MAXST);
      s.cps_q = wq ? (int)((nchq + wq - 1) / wq) : 1;
      s.nsq = wq ? (int)((nchq + s.cps_q - 1) / s.cps_q) : 0;
      s.cps_t = wt ? (int)((ncht + wt - 1) / wt) : 1;
      s.nst = wt ? (int)((ncht + s.cps_t - 1) / s.cps_t) : 0;
      if (s.nsq + s.nst == 0) s.nst = 1;  // empty sequence: one empty split writes zeros
      s.cta0 = cta;
      s.part0 = part;
      cta += hkv * (s.nsq + s.nst);
      part += hkv * (s.nsq + s.nst);
    }
    A.ncta = cta;
    // q / out rows are indexed by DecodeSeq::row, the workspace slots restart per launch
    if (dispatch(c->fam_k, c->bits_k, L, A, st) != cudaSuccess) return KVQ_E_CUDA;
    note_launches(1);
  }
  return KVQ_OK;
}

}  // namespace kvq
