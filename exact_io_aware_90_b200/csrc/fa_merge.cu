// fa_merge.cu — ring (context-parallel) attention's elementwise kernels.
//
// Merge of normalised partial attention results of the same queries over disjoint key sets
// (the block-merge rule of "FlashAttention 与算子融合", "FlashAttention 的两个关键", online softmax:
// m = max, ℓ = Σ ℓ_c·e^{m_c − m}, partial outputs scaled the same way), as ring / context-parallel
// attention produces them one block at a time.  A normalised part (O_b, LSE_b) is the pair
// (m, ℓ) = (LSE_b, 1) with Õ = O_b, so with m = max(LSE_acc, LSE_b):
//   LSE' = m + ln(e^{LSE_acc − m} + e^{LSE_b − m}),
//   O'   = e^{LSE_acc − LSE'}·O_acc + e^{LSE_b − LSE'}·O_b.
// Elementwise and HBM-bound: one thread per 8 features of one (token, head) row, 16-byte loads of the
// 16-bit part, 32-byte loads and stores of the fp32 accumulator.
#include "fa_internal.h"
#include "sm100.cuh"

#include <algorithm>

namespace fa {

template <bool BF16>
__global__ void __launch_bounds__(256) fa_merge_kernel(float* __restrict__ acc_o, float* __restrict__ acc_lse,
                                                        const uint4* __restrict__ part_o,
                                                        const float* __restrict__ part_lse, uint4* __restrict__ out,
                                                        long long rows, int d8, int first) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const bool valid = gid < rows * d8;
  const long long row = valid ? gid / d8 : 0;
  const int c8 = valid ? (int)(gid - row * d8) : 0;
  float wa = 0.f, wb = 1.f, l_new = 0.f;
  if (valid) {
    const float lb = part_lse[row];
    if (first) {
      l_new = lb;
    } else {
      const float la = acc_lse[row];
      const float m = fmaxf(la, lb);
      if (m == -INFINITY) {  // neither part saw a key: stays empty
        wa = 0.f;
        wb = 0.f;
        l_new = -INFINITY;
      } else {
        const float ea = __expf(la - m), eb = __expf(lb - m);  // e^{−∞} = 0 drops an empty part
        const float ell = ea + eb;
        l_new = m + __logf(ell);
        wa = ea / ell;
        wb = eb / ell;
      }
    }
  }
  // every thread of this row (d8 consecutive lanes of one warp) has read the old LSE before it is replaced
  __syncwarp();
  if (!valid) return;
  if (c8 == 0) acc_lse[row] = l_new;
  const uint4 pb = part_o[gid];
  const uint32_t pw[4] = {pb.x, pb.y, pb.z, pb.w};
  float o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = unpack2<BF16>(pw[i]);
    o[2 * i] = wb * f.x;
    o[2 * i + 1] = wb * f.y;
  }
  float4* acc4 = reinterpret_cast<float4*>(acc_o) + 2 * gid;
  if (!first) {
    const float4 a0 = acc4[0], a1 = acc4[1];
    const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = fmaf(wa, a[i], o[i]);
  }
  if (out != nullptr) {
    out[gid] = make_uint4(pack2<BF16>(o[0], o[1]), pack2<BF16>(o[2], o[3]), pack2<BF16>(o[4], o[5]),
                          pack2<BF16>(o[6], o[7]));
  } else {
    acc4[0] = make_float4(o[0], o[1], o[2], o[3]);
    acc4[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
}

// Gradient accumulation for the ring backward: acc (+)= part over n elements (8 per thread), where
// part is a dtype gradient partial (NULL: nothing added); with `out` the sum is written there in the
// dtype instead of back into acc.  Elementwise, HBM-bound.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_accum_kernel(float4* __restrict__ acc, const uint4* __restrict__ part,
                                                        uint4* __restrict__ out, long long n8, int first) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (!first) {
      const float4 a0 = acc[2 * i], a1 = acc[2 * i + 1];
      v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w;
      v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
    }
    if (part != nullptr) {
      const uint4 pb = part[i];
      const uint32_t pw[4] = {pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = unpack2<BF16>(pw[k]);
        v[2 * k] += f.x;
        v[2 * k + 1] += f.y;
      }
    }
    if (out != nullptr) {
      out[i] = make_uint4(pack2<BF16>(v[0], v[1]), pack2<BF16>(v[2], v[3]), pack2<BF16>(v[4], v[5]),
                          pack2<BF16>(v[6], v[7]));
    } else {
      acc[2 * i] = make_float4(v[0], v[1], v[2], v[3]);
      acc[2 * i + 1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

cudaError_t launch_accumulate(float* acc, const void* part, void* out, long long n, bool bf16, int first,
                              cudaStream_t stream) {
  const long long n8 = n / 8;
  const unsigned blocks = (unsigned)std::min<long long>((n8 + 255) / 256, 148LL * 16);
  if (bf16)
    fa_accum_kernel<true><<<blocks, 256, 0, stream>>>(reinterpret_cast<float4*>(acc),
                                                      reinterpret_cast<const uint4*>(part),
                                                      reinterpret_cast<uint4*>(out), n8, first);
  else
    fa_accum_kernel<false><<<blocks, 256, 0, stream>>>(reinterpret_cast<float4*>(acc),
                                                       reinterpret_cast<const uint4*>(part),
                                                       reinterpret_cast<uint4*>(out), n8, first);
  return cudaPeekAtLastError();
}

cudaError_t launch_merge(float* acc_o, float* acc_lse, const void* part_o, const float* part_lse, void* out,
                         long long rows, int d, bool bf16, int first, cudaStream_t stream) {
  const int d8 = d / 8;
  const long long n = rows * d8;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (bf16)
    fa_merge_kernel<true><<<blocks, 256, 0, stream>>>(acc_o, acc_lse, reinterpret_cast<const uint4*>(part_o),
                                                      part_lse, reinterpret_cast<uint4*>(out), rows, d8, first);
  else
    fa_merge_kernel<false><<<blocks, 256, 0, stream>>>(acc_o, acc_lse, reinterpret_cast<const uint4*>(part_o),
                                                       part_lse, reinterpret_cast<uint4*>(out), rows, d8, first);
  return cudaPeekAtLastError();
}

}  // namespace fa
