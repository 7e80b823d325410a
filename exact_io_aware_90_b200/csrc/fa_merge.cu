// fa_merge.cu — merge of normalised partial attention results of the same queries over disjoint key sets
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
