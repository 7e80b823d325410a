// fa_decode.cu — token-by-token decoding with split-KV for sm_100a.
//
// One new query token per sequence attends to all keys of its sequence (the
// K/V cache).  The pages set this workload apart ("FlashAttention 短片讲解稿",
// segment "适用范围与关键结论": decoding has a different shape, its benefit has
// to be measured): with a single query row the work is a stream over the
// cache, bound by HBM bandwidth, not by the tensor cores, so these kernels run
// on the CUDA cores with wide streaming loads.
//
//   fa_decode_split_kernel  one CTA per (sequence, head, chunk of 512 keys):
//                           partial (m, ℓ, Õ = Σ_j 2^(s_j − m) v_j) of the
//                           chunk, s = scale·log2(e)·q·k (base 2)
//   fa_decode_merge_kernel  one CTA per (sequence, head): merges the chunks
//                           ("FlashAttention 与算子融合", "FlashAttention 的两个
//                           关键": m = max m_c, ℓ = Σ ℓ_c·2^(m_c − m), and the
//                           partial outputs scaled the same way), writes
//                           O = Õ/ℓ and LSE = (m + log2 ℓ)·ln 2
//
// Split kernel layout: 8 warps × 64 keys.  A lane holds 16 features of q and of
// the output; d/16 consecutive lanes (a lane group) work on one key, so a warp
// covers 32·16/d keys at a time, 4 per lane group per step (the running max and
// the rescale of the partial output are done once per 4 keys).  Lane groups are
// merged with shuffles, warps through shared memory.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

constexpr int kDecThreads = 256;  // 8 warps
constexpr int kDecWarpKeys = kDecChunkKeys / 8;
constexpr int kDecStep = 4;  // keys per lane group between two rescales

struct DecParams {
  const uint8_t* q;
  const uint8_t* k;
  const uint8_t* v;
  void* o;
  float* lse;
  float* part_o;   // [B·H, nchunk, d]
  float* part_ml;  // [B·H, nchunk, 2]: m (base-2 scaled domain), ℓ
  const int32_t* cu_seqlens_k;
  int B, H, Nk, Tk, nchunk;
  float scale_log2;
};

__device__ __forceinline__ bool dec_segment(const DecParams& p, int b, int& tok0, int& L) {
  if (p.cu_seqlens_k != nullptr) {
    tok0 = __ldg(p.cu_seqlens_k + b);
    const int end = __ldg(p.cu_seqlens_k + b + 1);
    L = end - tok0;
    if (tok0 < 0 || L < 0 || end > p.Tk || L > p.Nk) {
      record_status(1);
      return false;
    }
  } else {
    tok0 = b * p.Nk;
    L = p.Nk;
  }
  return true;
}

// 16 features (32 bytes) of one row, as 8 packed pairs, streamed (read once).
__device__ __forceinline__ void ld_row16(const uint8_t* ptr, uint32_t (&r)[8]) {
  const uint4 a = __ldcs(reinterpret_cast<const uint4*>(ptr));
  const uint4 b = __ldcs(reinterpret_cast<const uint4*>(ptr) + 1);
  r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
  r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
}

// Merges partial (m, ℓ, o[16]) of another lane into this lane's.
__device__ __forceinline__ void dec_merge(float& m, float& l, float2 (&o)[8], float m2, float l2, const float2 (&o2)[8]) {
  const float mn = fmaxf(m, m2);
  const float a = (m == -INFINITY) ? 0.f : ex2(m - mn);
  const float a2 = (m2 == -INFINITY) ? 0.f : ex2(m2 - mn);
  l = l * a + l2 * a2;
  const float2 aa = make_float2(a, a), bb = make_float2(a2, a2);
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = __ffma2_rn(o2[i], bb, __fmul2_rn(o[i], aa));
  m = mn;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kDecThreads) fa_decode_split_kernel(const DecParams p) {
  constexpr int G = D / 16;      // lanes per key
  constexpr int KPW = 32 / G;    // keys per warp at a time
  __shared__ float s_ml[8][2];
  __shared__ float2 s_o[8][D / 2];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  int tok0, L;
  if (!dec_segment(p, b, tok0, L)) return;
  const int c0 = c * kDecChunkKeys;
  if (c0 >= L) return;  // the merge reads only the chunks inside the sequence
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / G, r = lane % G;  // lane group (key), feature slice [16r, 16r + 16)
  // q · scale·log2(e), 16 features
  float2 q2[8];
  {
    uint32_t qr[8];
    ld_row16(p.q + (((size_t)b * p.H + h) * D + 16 * r) * 2, qr);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = unpack2<BF16>(qr[i]);
      q2[i] = make_float2(f.x * p.scale_log2, f.y * p.scale_log2);
    }
  }
  float m = -INFINITY, l = 0.f;
  float2 o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = make_float2(0.f, 0.f);
  const size_t row_stride = (size_t)p.H * D * 2;
  const uint8_t* kbase = p.k + (((size_t)tok0) * p.H + h) * D * 2 + 32 * r;
  const uint8_t* vbase = p.v + (((size_t)tok0) * p.H + h) * D * 2 + 32 * r;
  const int wk0 = c0 + warp * kDecWarpKeys;  // this warp's first key
#pragma unroll 1
  for (int j0 = wk0; j0 < wk0 + kDecWarpKeys && j0 < L; j0 += KPW * kDecStep) {
    // keys j0 + grp + KPW·u, u = 0..kDecStep-1, for this lane group
    uint32_t kr[kDecStep][8], vr[kDecStep][8];
#pragma unroll
    for (int u = 0; u < kDecStep; ++u) {
      const int j = j0 + grp + KPW * u;
      if (j < L && j < wk0 + kDecWarpKeys) {
        ld_row16(kbase + (size_t)j * row_stride, kr[u]);
        ld_row16(vbase + (size_t)j * row_stride, vr[u]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) kr[u][i] = vr[u][i] = 0u;
      }
    }
    float s[kDecStep];
#pragma unroll
    for (int u = 0; u < kDecStep; ++u) {
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = __ffma2_rn(q2[i], unpack2<BF16>(kr[u][i]), acc);
      float dot = acc.x + acc.y;
#pragma unroll
      for (int off = G / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const int j = j0 + grp + KPW * u;
      s[u] = (j < L && j < wk0 + kDecWarpKeys) ? dot : -INFINITY;
    }
    float smax = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
    const float mn = fmaxf(m, smax);
    if (mn != -INFINITY) {
      const float a = (m == -INFINITY) ? 0.f : ex2(m - mn);
      const float2 aa = make_float2(a, a);
      l *= a;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = __fmul2_rn(o[i], aa);
#pragma unroll
      for (int u = 0; u < kDecStep; ++u) {
        const float pu = ex2(s[u] - mn);  // 0 for a key outside the sequence
        l += pu;
        const float2 pp = make_float2(pu, pu);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = __ffma2_rn(pp, unpack2<BF16>(vr[u][i]), o[i]);
      }
      m = mn;
    }
  }
  // lane groups of the warp: lanes with the same feature slice hold partials of different keys
#pragma unroll
  for (int off = G; off < 32; off <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
    float2 o2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o2[i].x = __shfl_xor_sync(0xffffffffu, o[i].x, off);
      o2[i].y = __shfl_xor_sync(0xffffffffu, o[i].y, off);
    }
    dec_merge(m, l, o, m2, l2, o2);
  }
  // warps: lane group 0 of each warp publishes, warp 0 merges the 8
  if (grp == 0) {
    if (r == 0) {
      s_ml[warp][0] = m;
      s_ml[warp][1] = l;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) s_o[warp][8 * r + i] = o[i];
  }
  __syncthreads();
  if (warp == 0 && grp == 0) {
    m = s_ml[0][0];
    l = s_ml[0][1];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = s_o[0][8 * r + i];
    for (int w = 1; w < 8; ++w) {
      float2 o2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o2[i] = s_o[w][8 * r + i];
      dec_merge(m, l, o, s_ml[w][0], s_ml[w][1], o2);
    }
    const size_t slot = ((size_t)b * p.H + h) * p.nchunk + c;
    float4* po = reinterpret_cast<float4*>(p.part_o + slot * D + 16 * r);
#pragma unroll
    for (int i = 0; i < 4; ++i) po[i] = make_float4(o[2 * i].x, o[2 * i].y, o[2 * i + 1].x, o[2 * i + 1].y);
    if (r == 0) {
      p.part_ml[slot * 2] = m;
      p.part_ml[slot * 2 + 1] = l;
    }
  }
}

// One CTA of D threads per (sequence, head); thread = feature.
template <int D, bool BF16>
__global__ void __launch_bounds__(D) fa_decode_merge_kernel(const DecParams p) {
  const int h = blockIdx.x, b = blockIdx.y, f = threadIdx.x;
  int tok0, L;
  if (!dec_segment(p, b, tok0, L)) return;
  const int nc = (L + kDecChunkKeys - 1) / kDecChunkKeys;
  const size_t base = ((size_t)b * p.H + h) * p.nchunk;
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, p.part_ml[(base + c) * 2]);
  float ell = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int c = 0; c < nc; ++c) {
      const float mc = p.part_ml[(base + c) * 2];
      const float w = (mc == -INFINITY) ? 0.f : ex2(mc - M);
      ell = fmaf(p.part_ml[(base + c) * 2 + 1], w, ell);
      acc = fmaf(p.part_o[(base + c) * D + f], w, acc);
    }
  }
  const float out = (ell > 0.f) ? acc / ell : 0.f;
  const size_t oi = ((size_t)b * p.H + h) * D + f;
  if constexpr (BF16) reinterpret_cast<__nv_bfloat16*>(p.o)[oi] = __float2bfloat16_rn(out);
  else reinterpret_cast<__half*>(p.o)[oi] = __float2half_rn(out);
  if (f == 0) p.lse[(size_t)b * p.H + h] = (ell > 0.f) ? (M + __log2f(ell)) * 0.69314718055994531f : -INFINITY;
}

template <int D, bool BF16>
static cudaError_t launch_decode_t(const Problem& pb, const DecodeArgs& a, cudaStream_t stream) {
  DecParams p;
  p.q = static_cast<const uint8_t*>(a.q);
  p.k = static_cast<const uint8_t*>(a.k);
  p.v = static_cast<const uint8_t*>(a.v);
  p.o = a.o;
  p.lse = a.lse;
  p.part_o = a.part_o;
  p.part_ml = a.part_ml;
  p.cu_seqlens_k = pb.cu_seqlens;
  p.B = pb.B;
  p.H = pb.H;
  p.Nk = pb.N;
  p.Tk = pb.T;
  p.nchunk = decode_chunks(pb.N);
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  fa_decode_split_kernel<D, BF16><<<dim3((unsigned)p.nchunk, (unsigned)pb.H, (unsigned)pb.B), kDecThreads, 0, stream>>>(p);
  cudaError_t e = cudaPeekAtLastError();
  if (e != cudaSuccess) return e;
  fa_decode_merge_kernel<D, BF16><<<dim3((unsigned)pb.H, (unsigned)pb.B), D, 0, stream>>>(p);
  return cudaPeekAtLastError();
}

cudaError_t launch_decode(const Problem& pb, const DecodeArgs& a, cudaStream_t stream) {
  if (pb.d == 128) return pb.bf16 ? launch_decode_t<128, true>(pb, a, stream) : launch_decode_t<128, false>(pb, a, stream);
  return pb.bf16 ? launch_decode_t<64, true>(pb, a, stream) : launch_decode_t<64, false>(pb, a, stream);
}

}  // namespace fa
