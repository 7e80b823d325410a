// fa_internal.h — declarations shared by the host-side entry points and the
// kernel launchers of libfa_b200.so (not part of the public ABI).
#pragma once

#include <cstddef>
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

// Dropout on P: element (query i, key j) of the sequence/head with global index bh = b·H + h is kept
// when byte (j mod 4) of word (i mod 4) of Philox(counter (j/4, i/4, bh, offset), key = seed) is at
// least `t`; kept elements are scaled by keep_scale = 256/(256 − t).
struct Dropout {
  uint32_t t;         // threshold byte (0 = no dropout)
  float keep_scale;
  uint32_t seed_lo, seed_hi;
  uint32_t offset;
};

// Raises a kernel's dynamic shared-memory limit on the current device once per device: the attribute
// belongs to the device's context, so a process driving several GPUs sets it on each.  `done` holds
// one bit per device ordinal (ordinals from 64 on set it on every call).
inline cudaError_t set_smem_once(std::atomic<unsigned long long>& done, const void* kern, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit != 0ull && (done.load(std::memory_order_acquire) & bit) != 0ull) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Work of one attention call, resolved on the host.
struct Problem {
  int B, H, N, d, T;
  float scale;
  int causal;
  const int32_t* cu_seqlens;  // device pointer or nullptr
  bool bf16;
  uint64_t timeout_ns;
  Dropout drop;  // drop.t == 0: no dropout
  // e4m3 inputs (forward only; output bf16): real value = stored value × descale
  bool fp8;
  float qk_descale;  // q descale × k descale
  float v_descale;
  // or one descale per (sequence, head): fp32 [B·H] device arrays (nullptr: per tensor), or, when
  // descale_blocks > 0, one per (128-token block, head): fp32 [descale_blocks·H] device arrays
  const float* q_descale_bh;
  const float* k_descale_bh;
  const float* v_descale_bh;
  int descale_blocks;
};

struct FwdArgs {
  CUtensorMap tm_q, tm_k, tm_v;
  void* o;
  float* lse;
};

struct BwdArgs {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  CUtensorMap tm_dq;  // the fp32 dQ accumulator, for TMA reduce-add
  const void* q;
  const void* k;
  const float* lse;
  const void* o;
  const void* dO;
  void* dq;
  void* dk;
  void* dv;
  float* dq_acc;  // [T, H, d] fp32
  float* delta;   // [T, H] fp32
};

// Encodes a [T, H, d] 16-bit tensor as a 3-D TMA map with 128-byte swizzle
// and a box of 64 features × 1 head × `rows` tokens.  Returns false on failure.
bool encode_tmap(CUtensorMap* map, const void* base, int T, int H, int d, bool bf16, int rows);

// Encodes a [T, H, d] fp32 tensor as a 3-D TMA map with 128-byte swizzle and a
// box of 32 features × 1 head × `rows` tokens.  Returns false on failure.
bool encode_tmap_e4m3(CUtensorMap* map, const void* base, int T, int H, int d, int rows);
bool encode_tmap_f32(CUtensorMap* map, const void* base, int T, int H, int d, int rows);

// Decode (one query per sequence, split-KV): keys per chunk, and its workspace.
constexpr int kDecChunkKeys = 512;
inline int decode_chunks(int Nk) { return (Nk + kDecChunkKeys - 1) / kDecChunkKeys; }
struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  float* part_o;   // [B·H, chunks, d] fp32
  float* part_ml;  // [B·H, chunks, 2] fp32
};

cudaError_t launch_fwd(const Problem& pb, const FwdArgs& a, cudaStream_t stream);
// Merge of a normalised partial (O_b, LSE_b) into an fp32 running result over rows = T·H (fa_merge.cu).
cudaError_t launch_merge(float* acc_o, float* acc_lse, const void* part_o, const float* part_lse, void* out,
                         long long rows, int d, bool bf16, int first, cudaStream_t stream);

// acc (+)= part over n elements (n a multiple of 8), optionally written to `out` in the dtype (fa_merge.cu).
cudaError_t launch_accumulate(float* acc, const void* part, void* out, long long n, bool bf16, int first,
                              cudaStream_t stream);

cudaError_t launch_decode(const Problem& pb, const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_pre(const Problem& pb, const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_main(const Problem& pb, const BwdArgs& a, cudaStream_t stream);
int bwd_q_tile_rows(int d, bool dropout);
int bwd_dq_box_rows(int d, bool dropout);
cudaError_t launch_bwd_post(const Problem& pb, const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_watchdog_selftest(uint64_t timeout_ns, cudaStream_t stream);

}  // namespace fa
