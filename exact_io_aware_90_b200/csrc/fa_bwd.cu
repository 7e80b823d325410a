// fa_bwd.cu — attention backward for sm_100a.
//
// The forward keeps only O and the row log-sum-exp; the backward recomputes
// the probabilities tile by tile from Q, K and the LSE ("FlashAttention
// 短片讲解稿", segment "第三招 · 反向重计算").  The gradient equations are the
// chain rule of the forward definition:
//   P = exp(scale·QKᵀ − LSE),  dV = Pᵀ dO,  dP = dO Vᵀ,  D_i = Σ_c dO_ic O_ic,
//   dS = P ∘ (dP − D),  dQ = scale·dS K,  dK = scale·dSᵀ Q.
//
// Three kernels on one stream:
//   fa_bwd_pre_kernel        D (fp32 [T, H]) and a zeroed fp32 dQ accumulator
//   fa_bwd_main_q128_kernel  work unit = (sequence, head, 128-key tile j), run by persistent CTAs:
//                            K_j, V_j stay in shared memory; Q_i, dO_i (128 query rows per
//                            step) stream in.  Per step:
//                              Sᵀ  = K_j Q_iᵀ, dPᵀ = V_j dO_iᵀ      (tensor memory, fp32)
//                              Pᵀ  = 2^(c·Sᵀ − LSE_i·log2 e), masked (two compute warpgroups)
//                              dV += Pᵀ dO_i                          (Pᵀ read from tensor memory)
//                              dSᵀ = Pᵀ ∘ (dPᵀ − D_i)
//                              dK += dSᵀ Q_i                          (dSᵀ read from tensor memory)
//                              dQ_i partial = dS K_j                  (dSᵀ staged in shared memory)
//                            and the dQ warpgroup stages the partial in shared memory, from where
//                            TMA reduce-adds it into the fp32 accumulator.  dK (× scale) and dV
//                            are written once per unit.  With dropout the keep mask of each
//                            (query, key) is regenerated from the same Philox stream as the
//                            forward: dV takes the dropped Pᵀ (its 1/(1 − p) applied at the end)
//                            and dSᵀ = Pᵀ ∘ (Z ∘ dPᵀ / (1 − p) − D).
//   fa_bwd_post_kernel       dq = scale · accumulator, rounded to the dtype
// All five MMAs are 128 × 128 × d or 128 × d × 128 (full tensor-core rate): at d = 128 the dQ product
// is formed transposed, dQᵀ = K_jᵀ dSᵀ (M = d), at d = 64 directly (M = 128 queries).
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

// ============================================================================ preprocess / postprocess

// One thread per 8 features of one (token, head) row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dO,
                                                         float* __restrict__ delta, float4* __restrict__ dq_acc,
                                                         long long rows) {
  constexpr int TPR = D / 8;  // threads per row
  const long long n = rows * TPR;
  const int lane = threadIdx.x & 31;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  // whole warps step together so the row reduction below always has 32 lanes
  for (long long base = warp0 * 32; base < n; base += nwarps * 32) {
    const long long idx = base + lane;
    const bool live = idx < n;
    float acc = 0.f;
    if (live) {
      const uint4 a = __ldg(o + idx);
      const uint4 g = __ldg(dO + idx);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 fa, fg;
        if constexpr (BF16) {
          fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[i]));
          fg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv[i]));
        } else {
          fa = __half22float2(*reinterpret_cast<const __half2*>(&av[i]));
          fg = __half22float2(*reinterpret_cast<const __half2*>(&gv[i]));
        }
        acc = fmaf(fa.x, fg.x, acc);
        acc = fmaf(fa.y, fg.y, acc);
      }
    }
    // reduce over the TPR consecutive lanes of this row (TPR divides 32, rows start at multiples of TPR)
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (live) {
      if ((lane % TPR) == 0) delta[idx / TPR] = acc;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      dq_acc[2 * idx] = z;
      dq_acc[2 * idx + 1] = z;
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_post_kernel(const float4* __restrict__ dq_acc, uint2* __restrict__ dq,
                                                          long long n4, float scale, const int32_t* cu_seqlens,
                                                          int B, long long row_elems4) {
  long long limit = n4;
  if (cu_seqlens != nullptr) limit = min(n4, (long long)__ldg(cu_seqlens + B) * row_elems4);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < limit; i += (long long)gridDim.x * blockDim.x) {
    const float4 a = dq_acc[i];
    uint2 out;
    out.x = pack2<BF16>(a.x * scale, a.y * scale);
    out.y = pack2<BF16>(a.z * scale, a.w * scale);
    dq[i] = out;
  }
}

// ============================================================================ main kernel

struct BwdParams {
  const float* lse;
  const float* delta;
  float* dq_acc;
  void* dk;
  void* dv;
  const int32_t* cu_seqlens;
  int B, H, N, T;
  int causal;
  int num_kblocks;  // ceil(N / 128)
  int heads_group;
  float scale;
  float scale_log2;
  uint64_t timeout_ns;
  Dropout drop;
};

constexpr int kBK = 128;  // keys per CTA

__device__ __forceinline__ void drain_wait_b(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      record_status(4);
      return;
    }
  }
}

__device__ __forceinline__ bool warp_wait_b(uint32_t bar, uint32_t parity, const Watchdog& wd) {
  const bool ok = mbar_wait(bar, parity, wd);
  return __all_sync(0xffffffffu, ok);
}

// Warp-uniform non-blocking probe of one barrier phase.
__device__ __forceinline__ bool warp_test_b(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_test_wait(bar, parity));
}

// Products of one Q tile, issued by one elected lane.  Descriptor arguments
// are pre-built bases; per 16-element K step only a constant start-address
// offset (16-byte units) is added.
// Sᵀ = K Qᵀ and dPᵀ = V dOᵀ: A = K or V (K-major, 128 rows), B = Q or dO
// (K-major, BQ rows); K dim = d.
template <int D, int BQ, uint32_t IDESC>
__device__ __forceinline__ void bwd_issue_kt(uint32_t d_tmem, uint64_t da, uint64_t db) {
  da = opaque64(da);
  db = opaque64(db);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t oa = ((kk >> 2) * (kBK * 128) + (kk & 3) * 32) >> 4;
    const uint32_t ob = ((kk >> 2) * (BQ * 128) + (kk & 3) * 32) >> 4;
    mma_ss(d_tmem, da + oa, db + ob, IDESC, kk > 0 ? 1u : 0u);
  }
}

// dV += Pᵀ dO or dK += dSᵀ Q: A from tensor memory (8 packed columns per step),
// B = dO or Q MN-major (+2 KB per 16 query rows); K dim = BQ.
template <int BQ, uint32_t IDESC>
__device__ __forceinline__ void bwd_issue_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t db, uint32_t acc) {
  db = opaque64(db);
#pragma unroll
  for (int kk = 0; kk < BQ / 16; ++kk) mma_ts(d_tmem, a_tmem + kk * 8, db + ((kk * 2048) >> 4), IDESC, kk > 0 ? 1u : acc);
}

// ============================================================================ main kernel, 128-query steps
//
// Every Q step covers 128 query rows, so the score, dP, dV, dK and dQ products are all 128 × 128 × 128
// at d = 128 (N = 128: at N = 64 the tensor core is starved by its shared-memory operand reads).  Two
// compute warpgroups form Pᵀ and dSᵀ concurrently, one per 64-query half of the step (thread = key
// row).  Tensor memory cannot hold Sᵀ and
// dPᵀ of a step beside dK and dV (128 columns each) plus a dQ partial, so columns are reused:
//   [0, 128)    Sᵀ(j); once both halves are in registers, dQᵀ(j − 1) = Kᵀ dSᵀ(j − 1) [128 features ×
//               128 queries]; once that has been read out, Pᵀ(j) packed into [0, 64) (half a in
//               [32a, 32a + 32))
//   [128, 256)  dPᵀ(j); once both halves are in registers, dSᵀ(j) packed into [128, 192)
//   [256, 384)  dK,  [384, 512)  dV
// The two warpgroups tell each other "my half of Sᵀ (dPᵀ) is in registers" through an mbarrier before
// anything is written over the other half's columns.  MMA issue order per step j (one thread; tcgen05
// MMAs of one thread run in issue order, so each product has read its tensor-memory operand before a
// later one overwrites it):
//   dV(j) after Pᵀ(j); Sᵀ(j + 1) right behind it (so it is computed while dSᵀ(j) is formed); dK(j)
//   after dSᵀ(j); dQᵀ(j) once Sᵀ(j + 1) has been read; dPᵀ(j + 1).
// The dQ partial goes from tensor memory to the fp32 accumulator through shared memory: the dQ
// warpgroup takes the whole partial into registers at once (so [0, 128) is released early), then each
// of its warps stages 32 features × 32 queries at a time as one TMA box (two boxes per warp, used in
// turn) and adds it into the accumulator with a TMA reduce-add (per-thread red.global.add of the same
// data measured far slower).
constexpr int kBwd128Threads = 512;  // 4 warpgroups
// Column pairs i (of 32 per 64-query half) with bit (i % 8) set take the FMA-pipe exp2 polynomial in
// the Pᵀ phase.  At d = 64 the compute phases set the step (the products take ~1.3k cycles of it), and a
// quarter of the exponentials there measured ~2 % faster; at d = 128 it measured slower.
template <int D> struct BwdPolyMask { static constexpr uint32_t value = 0x00u; };
template <> struct BwdPolyMask<64> { static constexpr uint32_t value = 0x22u; };

template <int D>
struct Bq128 {
  static constexpr int BQ = 128;
  static constexpr int NCH = D / 64;           // 64-feature (128-byte) chunks per row
  static constexpr uint32_t CHUNK = 128 * 128;  // [128 rows × 64 features], 128-byte swizzle
  static constexpr uint32_t TILE = NCH * CHUNK;  // [128 rows × D features]
  // d = 64: dQ (= dS K, lane = query) has tensor-memory columns of its own; d = 128: dQᵀ (= Kᵀ dSᵀ,
  // lane = feature) is written over Sᵀ once the next Sᵀ is in registers
  static constexpr bool DQ_OWN = (D == 64);
  // tensor memory columns
  static constexpr uint32_t T_S = 0, T_P = 0, T_DP = 128, T_DS = 128, T_DK = 256, T_DV = 256 + D;
  static constexpr uint32_t T_DQ = DQ_OWN ? 256 + 2 * D : 0;
  // barriers
  static constexpr int B_KVFULL = 0;    // K, V of the unit landed
  static constexpr int B_KVEMPTY = 1;   // K, V no longer read (the unit's last MMAs done)
  static constexpr int B_QFULL = 2;     // [2] Q tile of stage s landed
  static constexpr int B_QEMPTY = 4;    // [2] Q tile and row terms of stage s no longer read
  static constexpr int B_ROWFULL = 6;   // [2] −LSE·log2 e and −D of stage s written (32 arrivals)
  static constexpr int B_DOFULL = 8;
  static constexpr int B_DOEMPTY = 9;
  static constexpr int B_SFULL = 10;
  static constexpr int B_DPFULL = 11;
  static constexpr int B_SREAD = 12;    // both halves of Sᵀ in registers (256 arrivals)
  static constexpr int B_DPREAD = 13;   // both halves of dPᵀ in registers (256 arrivals)
  static constexpr int B_PREADY = 14;   // [2] half a of Pᵀ in tensor memory (128 arrivals)
  static constexpr int B_DSREADY = 16;  // [2] half a of dSᵀ in tensor and shared memory (128 arrivals)
  static constexpr int B_DQFULL = 18;
  static constexpr int B_DQFREE = 19;   // the dQ partial read out of tensor memory (128 arrivals)
  static constexpr int B_DKV = 20;      // dK, dV of the unit complete
  static constexpr int B_DKVFREE = 21;  // dK, dV read out of tensor memory (128 arrivals)
  static constexpr int B_UFULL = 22;    // [2] work-unit ring slot written
  static constexpr int B_UEMPTY = 24;   // [2] slot read by every reader warp
  static constexpr int B_CLC = 26;      // scheduler response landed
  static constexpr int B_DRAIN = 27;
  static constexpr int NBARS = 28;
  static constexpr int UNIT_READERS = 14;  // compute warps 0-7, dQ warps 8-11, MMA warp 13, row-term warp 14
  // shared memory: K, V resident; Q double-buffered; dO single (its next tile loads once dV has read
  // it, well before the next dPᵀ); dSᵀ as two [128 keys × 64 queries] chunks (operand of the dQ product)
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = TILE;
  static constexpr uint32_t OFF_Q = 2 * TILE;
  static constexpr uint32_t OFF_DO = 4 * TILE;
  static constexpr uint32_t OFF_DS = 5 * TILE;
  static constexpr uint32_t OFF_DQS = OFF_DS + 2 * CHUNK;  // dQ staging: per dQ warp two boxes [32 rows × 32 fp32]
  static constexpr uint32_t DQ_BOX = 32 * 128;
  static constexpr uint32_t OFF_ROW = OFF_DQS + 8 * DQ_BOX;  // per stage: −LSE·log2 e [128], −D [128] (fp32)
  static constexpr uint32_t OFF_CLC = OFF_ROW + 2 * 2 * BQ * 4;  // 16-byte scheduler response
  static constexpr uint32_t OFF_BAR = OFF_CLC + 16;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;  // TMEM base, abort flag, unit ring [2]
  // no alignment slack: the dynamic shared memory is declared 1024-byte aligned (checked at run time)
  static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // registers per thread after setmaxnreg: the block is launched at 128 (512 threads), so the four
  // warpgroups' shares must add up to at most 4 × 128
  static constexpr uint32_t REGS_LAUNCH = 128;  // 65536 registers / 512 threads (ptxas reports 128)
  static constexpr uint32_t REGS_CMP = 152, REGS_DQ = 152, REGS_IO = 56;
  static_assert(2 * REGS_CMP + REGS_DQ + REGS_IO <= 4 * REGS_LAUNCH, "register budget");
};

// dQᵀ = Kᵀ dSᵀ: A = K MN-major (M = 128 features), B = dSᵀ MN-major (N = 128 queries, two 64-query
// chunks 16 KB apart), K dim = the 128 keys (+2 KB per 16 keys in both operands).
template <uint32_t IDESC>
__device__ __forceinline__ void bwd_issue_dq128(uint32_t d_tmem, uint64_t da, uint64_t db) {
  da = opaque64(da);
  db = opaque64(db);
#pragma unroll
  for (int kk = 0; kk < kBK / 16; ++kk) mma_ss(d_tmem, da + ((kk * 2048) >> 4), db + ((kk * 2048) >> 4), IDESC, kk > 0 ? 1u : 0u);
}

// A decoded work unit of the backward: key tile [k0, k0 + 128) of the sequence whose tokens are
// [tok0, tok0 + L), head h; n_it Q steps from query tile i_begin.
struct BwdUnit {
  int tok0, L, k0, b, h, i_begin, n_it;
};

// Unit order: heads in groups (K, V, Q and dO of a group stay in L2), heaviest key tiles (the first
// ones when causal) first inside a group.  Returns false for a unit whose key tile lies past the end of
// its sequence; invalid sequence bounds are recorded as FA_ERR_INVALID_ARG (when `record`) and the
// unit is skipped.
__device__ __forceinline__ bool decode_bwd_unit(const BwdParams& p, int unit, BwdUnit& u, bool record) {
  const int BH = p.B * p.H;
  const int nkb = p.num_kblocks;
  const int G = p.heads_group;
  // Head groups run from the last (sequence, head) to the first: the preprocess kernel zeroes the dQ
  // accumulator in token order, so the last sequences' accumulator lines are the ones still in L2 when
  // this kernel starts, and the postprocess kernel, reading in token order, finds the lines this
  // kernel reduced into last still in L2.  A partial last group (fewer than G heads) comes first.
  const int full = BH / G, rem = BH - full * G;
  int group, g_heads, r;
  if (unit < rem * nkb) {
    group = full;
    g_heads = rem;
    r = unit;
  } else {
    const int u2 = unit - rem * nkb;
    group = full - 1 - u2 / (G * nkb);
    g_heads = G;
    r = u2 - (full - 1 - group) * G * nkb;
  }
  const int kb = r / g_heads;
  const int bh = group * G + r % g_heads;
  const int b = bh / p.H;
  u.b = b;
  u.h = bh - b * p.H;
  if (p.cu_seqlens != nullptr) {
    u.tok0 = __ldg(p.cu_seqlens + b);
    const int end = __ldg(p.cu_seqlens + b + 1);
    u.L = end - u.tok0;
    if (u.tok0 < 0 || u.L < 0 || end > p.T || u.L > p.N) {
      if (record) record_status(1);
      return false;
    }
  } else {
    u.tok0 = b * p.N;
    u.L = p.N;
  }
  u.k0 = kb * kBK;
  if (u.k0 >= u.L) return false;
  u.i_begin = p.causal ? u.k0 / 128 : 0;
  u.n_it = (u.L + 127) / 128 - u.i_begin;  // ≥ 1
  return true;
}

template <int D, bool BF16, bool DROP>
__global__ void __launch_bounds__(kBwd128Threads, 1)
    fa_bwd_main_q128_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = Bq128<D>;
  constexpr int BQ = C::BQ;
  constexpr uint32_t IDESC_ST = idesc_f16(BF16, kBK, BQ, false, false);  // Sᵀ = K Qᵀ, dPᵀ = V dOᵀ
  constexpr uint32_t IDESC_DKV = idesc_f16(BF16, kBK, D, false, true);   // dV += Pᵀ dO, dK += dSᵀ Q
  // d = 128: dQᵀ = Kᵀ dSᵀ (M = 128 features, N = 128 queries); d = 64: dQ = dS K (M = 128 queries,
  // N = 64 features); both operands MN-major
  constexpr uint32_t IDESC_DQ = C::DQ_OWN ? idesc_f16(BF16, BQ, D, true, true) : idesc_f16(BF16, D, BQ, true, true);

  extern __shared__ __align__(1024) uint8_t smem_aligned[];
  uint8_t* smem = smem_aligned;
  const uint32_t s_base = smem_u32(smem);
  if ((s_base & 1023u) != 0u) {  // the 128-byte-swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) record_status(2);
    return;
  }
  const uint32_t sK = s_base + C::OFF_K;
  const uint32_t sV = s_base + C::OFF_V;
  const uint32_t sQ = s_base + C::OFF_Q;
  const uint32_t sDO = s_base + C::OFF_DO;
  const uint32_t sDS = s_base + C::OFF_DS;
  const uint32_t clc_resp = s_base + C::OFF_CLC;
  float* row_buf = reinterpret_cast<float*>(smem + C::OFF_ROW);
  const uint32_t bar0 = s_base + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- set-up, once per CTA: the CTA then runs work units until none is left
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KVFULL), 1);
    mbar_init(bar(C::B_KVEMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::B_QFULL + s), 1);
      mbar_init(bar(C::B_QEMPTY + s), 1);
      mbar_init(bar(C::B_ROWFULL + s), 32);
      mbar_init(bar(C::B_PREADY + s), 128);
      mbar_init(bar(C::B_DSREADY + s), 128);
      mbar_init(bar(C::B_UFULL + s), 1);
      mbar_init(bar(C::B_UEMPTY + s), C::UNIT_READERS);
    }
    mbar_init(bar(C::B_DOFULL), 1);
    mbar_init(bar(C::B_DOEMPTY), 1);
    mbar_init(bar(C::B_SFULL), 1);
    mbar_init(bar(C::B_DPFULL), 1);
    mbar_init(bar(C::B_SREAD), 256);
    mbar_init(bar(C::B_DPREAD), 256);
    mbar_init(bar(C::B_DQFULL), 1);
    mbar_init(bar(C::B_DQFREE), 128);
    mbar_init(bar(C::B_DKV), 1);
    mbar_init(bar(C::B_DKVFREE), 128);
    mbar_init(bar(C::B_CLC), 1);
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, p.timeout_ns};

  // Reads the next unit from the ring (every reader warp; one lane arrives for the warp).
  uint32_t un = 0;  // units read by this warp
  auto read_unit = [&](int& unit) -> bool {
    const int s = un & 1;
    if (!warp_wait_b(bar(C::B_UFULL + s), (un >> 1) & 1, wd)) return false;
    unit = unit_ring[s];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(C::B_UEMPTY + s));
    __syncwarp();
    ++un;
    return true;
  };

  if (warp >= 12) {
    regs_set<C::REGS_IO, C::REGS_LAUNCH>();
    if (warp == 12) {
      // ================================================================ scheduler and TMA producer
      // Units come from the hardware scheduler: this CTA's own index first, then, one at a time, the
      // index of a CTA of the grid that has not started yet, whose launch is cancelled.  The next unit
      // is fetched while the current one is loaded, so that its K and V can be prefetched into L2.
      const uint64_t pol_kv = l2_policy_evict_first();
      const uint64_t pol_q = l2_policy_evict_last();
      uint32_t pub = 0;               // units published
      uint32_t kvn = 0, qn = 0, don = 0;  // K/V, Q and dO tiles loaded so far
      uint32_t c_issued = 0, c_done = 0;  // cancellation requests / responses
      bool can_steal = true, ok = true;
      auto steal = [&]() -> int {
        if (!can_steal) return -1;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(C::B_CLC), 16);
          clc_try_cancel(clc_resp, bar(C::B_CLC));
        }
        __syncwarp();
        ++c_issued;
        if (!warp_wait_b(bar(C::B_CLC), c_done & 1, wd)) {
          ok = false;
          return -1;
        }
        ++c_done;
        int x = -1;
        const bool got = clc_query(clc_resp, x);
        fence_proxy_async_smem();  // the read above before the next response overwrites it
        __syncwarp();
        if (!got) {
          can_steal = false;  // no CTA left; no further request may be made
          return -1;
        }
        return x;
      };
      // the next unit with work, from `unit` on (-1: none left)
      auto next_valid = [&](int unit, BwdUnit& u) -> int {
        while (unit >= 0 && !decode_bwd_unit(p, unit, u, true)) unit = steal();
        return unit;
      };
      auto publish = [&](int unit) -> bool {
        const int s = pub & 1;
        if (pub >= 2 && !warp_wait_b(bar(C::B_UEMPTY + s), ((pub >> 1) - 1) & 1, wd)) return false;
        if (elect_one()) {
          unit_ring[s] = unit;
          mbar_arrive(bar(C::B_UFULL + s));  // release: the store is visible once the phase flips
        }
        __syncwarp();
        ++pub;
        return true;
      };
      BwdUnit U, N;
      int cur = next_valid(blockIdx.x, U);
      while (ok && cur >= 0) {
        if (!publish(cur)) break;
        // K and V of this unit, once the previous unit's last MMAs have read the buffers
        if (kvn > 0 && !warp_wait_b(bar(C::B_KVEMPTY), (kvn - 1) & 1, wd)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(C::B_KVFULL), 2 * C::TILE);
          for (int c = 0; c < C::NCH; ++c) {
            tma_load_3d(sK + c * C::CHUNK, &tm_k, bar(C::B_KVFULL), c * 64, U.h, U.tok0 + U.k0, pol_kv);
            tma_load_3d(sV + c * C::CHUNK, &tm_v, bar(C::B_KVFULL), c * 64, U.h, U.tok0 + U.k0, pol_kv);
          }
        }
        __syncwarp();
        ++kvn;
        // the next unit, its K and V on their way into L2
        const int nxt = next_valid(steal(), N);
        if (nxt >= 0 && elect_one()) {
          for (int c = 0; c < C::NCH; ++c) {
            tma_prefetch_l2_3d(&tm_k, c * 64, N.h, N.tok0 + N.k0);
            tma_prefetch_l2_3d(&tm_v, c * 64, N.h, N.tok0 + N.k0);
          }
        }
        __syncwarp();
        for (int it = 0; ok && it < U.n_it; ++it) {
          const int i0 = (U.i_begin + it) * BQ;
          const int s = qn & 1;
          if (qn >= 2 && !warp_wait_b(bar(C::B_QEMPTY + s), ((qn >> 1) - 1) & 1, wd)) { ok = false; break; }
          if (elect_one()) {
            mbar_arrive_expect_tx(bar(C::B_QFULL + s), C::TILE);
            for (int c = 0; c < C::NCH; ++c)
              tma_load_3d(sQ + s * C::TILE + c * C::CHUNK, &tm_q, bar(C::B_QFULL + s), c * 64, U.h, U.tok0 + i0,
                          pol_q);
          }
          __syncwarp();
          ++qn;
          // dO of this step, once dV of the previous step has read the single buffer
          if (don > 0 && !warp_wait_b(bar(C::B_DOEMPTY), (don - 1) & 1, wd)) { ok = false; break; }
          if (elect_one()) {
            mbar_arrive_expect_tx(bar(C::B_DOFULL), C::TILE);
            for (int c = 0; c < C::NCH; ++c)
              tma_load_3d(sDO + c * C::CHUNK, &tm_do, bar(C::B_DOFULL), c * 64, U.h, U.tok0 + i0, pol_q);
          }
          __syncwarp();
          ++don;
        }
        cur = nxt;
        U = N;
      }
      if (ok) publish(-1);  // no unit left
      // Let every load and scheduler response this warp asked for land before the CTA can exit.
      if (elect_one()) {
        if (c_issued > c_done) drain_wait_b(bar(C::B_CLC), c_done & 1, p.timeout_ns);
        if (kvn > 0) drain_wait_b(bar(C::B_KVFULL), (kvn - 1) & 1, p.timeout_ns);
        for (uint32_t i = qn > 2 ? qn - 2 : 0u; i < qn; ++i)
          drain_wait_b(bar(C::B_QFULL + (i & 1)), (i >> 1) & 1, p.timeout_ns);
        if (don > 0) drain_wait_b(bar(C::B_DOFULL), (don - 1) & 1, p.timeout_ns);
      }
      __syncwarp();
    } else if (warp == 14) {
      // ================================================================ row terms
      // −LSE·log2 e and −D of each step's query rows into the stage of its Q tile (rows past the
      // sequence get 0).  A warp of its own: these strided loads would otherwise hold up the TMA issue.
      const float LOG2E = 1.4426950408889634f;
      uint32_t g = 0;  // steps so far (all units)
      int unit;
      while (read_unit(unit) && unit >= 0) {
        BwdUnit U;
        decode_bwd_unit(p, unit, U, false);
        bool ok = true;
        for (int it = 0; it < U.n_it; ++it, ++g) {
          const int s = g & 1;
          const int i0 = (U.i_begin + it) * BQ;
          if (g >= 2 && !warp_wait_b(bar(C::B_QEMPTY + s), ((g >> 1) - 1) & 1, wd)) { ok = false; break; }
          float* lse_s = row_buf + s * 2 * BQ;
          float* del_s = lse_s + BQ;
          for (int q = lane; q < BQ; q += 32) {
            const int qrow = i0 + q;
            const bool v = qrow < U.L;
            lse_s[q] = v ? -__ldg(p.lse + (size_t)(U.tok0 + qrow) * p.H + U.h) * LOG2E : 0.f;
            del_s[q] = v ? -__ldg(p.delta + (size_t)(U.tok0 + qrow) * p.H + U.h) : 0.f;
          }
          mbar_arrive(bar(C::B_ROWFULL + s));  // release: the stores above are visible to waiters
        }
        if (!ok) break;
      }
    } else if (warp == 13) {
      // ================================================================ MMA issuer
      const uint32_t tS = tmem + C::T_S, tP = tmem + C::T_P, tDQ = tmem + C::T_DQ, tDP = tmem + C::T_DP;
      const uint32_t tDS = tmem + C::T_DS, tDK = tmem + C::T_DK, tDV = tmem + C::T_DV;
      const uint64_t dK_kmaj = sdesc_sw128(sK, 16, 1024), dV_kmaj = sdesc_sw128(sV, 16, 1024);
      const uint64_t dQ_kmaj = sdesc_sw128(sQ, 16, 1024), dDO_kmaj = sdesc_sw128(sDO, 16, 1024);
      const uint64_t dQ_mn = sdesc_sw128(sQ, C::CHUNK, 1024), dDO_mn = sdesc_sw128(sDO, C::CHUNK, 1024);
      // dQ operands, both MN-major, +2 KB per 16 keys: d = 128: A = Kᵀ (features contiguous), B = dSᵀ
      // (queries contiguous, two 64-query chunks); d = 64: A = dS (queries contiguous), B = K
      const uint64_t dK_mn = sdesc_sw128(sK, C::CHUNK, 1024), dDS_mn = sdesc_sw128(sDS, C::CHUNK, 1024);
      const uint64_t dq_a = C::DQ_OWN ? dDS_mn : dK_mn, dq_b = C::DQ_OWN ? dK_mn : dDS_mn;
      constexpr uint32_t TILE16 = C::TILE >> 4;
      constexpr uint32_t HALF16 = (64 * 128) >> 4;  // 64 rows of a chunk: query half 1 of Q / dO
      uint32_t g = 0;   // steps so far (all units); step g uses Q stage g mod 2 and the g-th dO tile
      uint32_t u = 0;   // units so far
      bool ok = true;
      int unit;
      while (ok && read_unit(unit) && unit >= 0) {
        BwdUnit U;
        decode_bwd_unit(p, unit, U, false);
        // Sᵀ and dPᵀ of the unit's first step: K and V in shared memory; [0, 128) released by the read-out
        // of the previous unit's last dQᵀ ([128, 256) was read by its last dK, issued before)
        ok = warp_wait_b(bar(C::B_KVFULL), u & 1, wd) && warp_wait_b(bar(C::B_QFULL + (g & 1)), (g >> 1) & 1, wd) &&
             (C::DQ_OWN || g == 0 || warp_wait_b(bar(C::B_DQFREE), (g - 1) & 1, wd)) &&
             warp_wait_b(bar(C::B_DOFULL), g & 1, wd);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          bwd_issue_kt<D, BQ, IDESC_ST>(tS, dK_kmaj, dQ_kmaj + (g & 1) * TILE16);
          tc_commit(bar(C::B_SFULL));
          bwd_issue_kt<D, BQ, IDESC_ST>(tDP, dV_kmaj, dDO_kmaj);
          tc_commit(bar(C::B_DPFULL));
        }
        __syncwarp();
        // dK and dV of the previous unit must have been read out before this unit's first products
        // (accumulate = 0) overwrite them
        if (u > 0 && !warp_wait_b(bar(C::B_DKVFREE), (u - 1) & 1, wd)) { ok = false; break; }
        for (int it = 0; it < U.n_it; ++it, ++g) {
          const int s = g & 1;
          const bool more = it + 1 < U.n_it;
          const uint32_t g1 = g + 1;
          // dV += Pᵀ(a) dO(a), as each half of Pᵀ is formed
          if (!warp_wait_b(bar(C::B_PREADY + 0), g & 1, wd)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) bwd_issue_acc<64, IDESC_DKV>(tDV, tP, dDO_mn, it > 0 ? 1u : 0u);
          __syncwarp();
          if (!warp_wait_b(bar(C::B_PREADY + 1), g & 1, wd)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
            bwd_issue_acc<64, IDESC_DKV>(tDV, tP + 32u, dDO_mn + HALF16, 1u);
            tc_commit(bar(C::B_DOEMPTY));  // dO of this step is read by no later MMA
          }
          __syncwarp();
          // Sᵀ of the next step over [0, 128): Pᵀ there is read by the dV MMAs above, which run first, and
          // dQᵀ of the previous step has been read out
          if (more) {
            if (!warp_wait_b(bar(C::B_QFULL + (g1 & 1)), (g1 >> 1) & 1, wd) ||
                (!C::DQ_OWN && g > 0 && !warp_wait_b(bar(C::B_DQFREE), (g - 1) & 1, wd))) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              bwd_issue_kt<D, BQ, IDESC_ST>(tS, dK_kmaj, dQ_kmaj + (g1 & 1) * TILE16);
              tc_commit(bar(C::B_SFULL));
            }
            __syncwarp();
          }
          // dK += dSᵀ Q once both halves of dSᵀ are formed, and dQᵀ = Kᵀ dSᵀ over [0, 128) once both
          // halves of the next Sᵀ are in registers (a unit's last step: [0, 128) holds only Pᵀ, read by
          // its dV MMAs above).  dQᵀ goes first when it can: the next Pᵀ is written over [0, 64) only after
          // dQᵀ has been read out; otherwise dK fills the tensor core while the next Sᵀ is being read.
          if (!warp_wait_b(bar(C::B_DSREADY + 0), g & 1, wd) || !warp_wait_b(bar(C::B_DSREADY + 1), g & 1, wd)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // (d = 64: dQ has columns of its own, free once the previous dQ has been read out)
          const bool dq_first = C::DQ_OWN || !more || warp_test_b(bar(C::B_SREAD), g1 & 1);
          if (C::DQ_OWN && g > 0 && !warp_wait_b(bar(C::B_DQFREE), (g - 1) & 1, wd)) { ok = false; break; }
          if (dq_first) {
            tc_fence_after();
            if (elect_one()) {
              bwd_issue_dq128<IDESC_DQ>(tDQ, dq_a, dq_b);
              tc_commit(bar(C::B_DQFULL));
            }
            __syncwarp();
          }
          if (elect_one()) {
            bwd_issue_acc<BQ, IDESC_DKV>(tDK, tDS, dQ_mn + s * TILE16, it > 0 ? 1u : 0u);
            tc_commit(bar(C::B_QEMPTY + s));  // Q and row terms of this step no longer read
          }
          __syncwarp();
          if (!dq_first) {
            if (!warp_wait_b(bar(C::B_SREAD), g1 & 1, wd)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              bwd_issue_dq128<IDESC_DQ>(tDQ, dq_a, dq_b);
              tc_commit(bar(C::B_DQFULL));
            }
            __syncwarp();
          }
          // dPᵀ of the next step over [128, 256) (dSᵀ there is read by dK, issued above)
          if (more) {
            if (!warp_wait_b(bar(C::B_DOFULL), g1 & 1, wd)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              bwd_issue_kt<D, BQ, IDESC_ST>(tDP, dV_kmaj, dDO_kmaj);
              tc_commit(bar(C::B_DPFULL));
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        if (elect_one()) {
          tc_commit(bar(C::B_DKV));      // dK, dV of the unit complete
          tc_commit(bar(C::B_KVEMPTY));  // K and V no longer read
        }
        __syncwarp();
        ++u;
      }
      // every MMA issued so far must finish before tensor memory is released
      if (elect_one()) {
        tc_commit(bar(C::B_DRAIN));
        drain_wait_b(bar(C::B_DRAIN), 0, p.timeout_ns);
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    // ================================================================ Pᵀ / dSᵀ warpgroups (thread = key row)
    // warpgroup a forms query half a (64 queries) of each step
    regs_set<C::REGS_CMP, C::REGS_LAUNCH>();
    const int a = warp >> 2;
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t tS = tmem + lane_off + C::T_S + 64u * a;    // this half of Sᵀ
    const uint32_t tP = tmem + lane_off + C::T_P + 32u * a;    // this half of Pᵀ (packed)
    const uint32_t tDP = tmem + lane_off + C::T_DP + 64u * a;  // this half of dPᵀ
    const uint32_t tDS = tmem + lane_off + C::T_DS + 32u * a;  // this half of dSᵀ (packed, over dPᵀ)
    const int kr = 32 * quarter + lane;  // key row within the tile
    const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
    uint8_t* ds_row = smem + C::OFF_DS + a * C::CHUNK + kr * 128;
    const uint32_t keep_bias = keep_flag_bias(p.drop.t);  // used by the dropout variant only
    const uint32_t ks_bits = __float_as_uint(p.drop.keep_scale);
    uint32_t g = 0;  // steps so far (all units)
    bool ok = true;
    int unit;
    while (ok && read_unit(unit) && unit >= 0) {
      BwdUnit U;
      decode_bwd_unit(p, unit, U, false);
      const int key = U.k0 + kr;  // position in the sequence
      for (int it = 0; it < U.n_it; ++it, ++g) {
        const int i0 = (U.i_begin + it) * BQ + 64 * a;  // first query of this half
        const int s = g & 1;
        if (!warp_wait_b(bar(C::B_ROWFULL + s), (g >> 1) & 1, wd)) { ok = false; break; }
        const float* lse_h = row_buf + s * 2 * BQ + 64 * a;
        const float* del_h = lse_h + BQ;
        // visible queries for this key: q >= key (causal) and q < L; key < L
        const int q_lo = p.causal ? key - i0 : 0;    // first visible column of the half
        const int q_hi = (key < U.L) ? U.L - i0 : -1;  // one past the last visible column
        const bool full = __all_sync(0xffffffffu, q_lo <= 0 && q_hi >= 64);
        // dropout: the random bytes of this key for the half's 64 queries, word w = queries 4w .. 4w+3
        // (byte = query offset), the same Philox numbering as the forward.  One call covers the 4 keys
        // of a lane quad (key mod 4 = lane mod 4) × 4 queries: each lane of the quad makes 4 of the
        // half's 16 calls, reorders its call's bytes from (query word, key byte) to (key word, query
        // byte), and the quad exchanges words.  Made before Sᵀ is read, while the registers are free.
        uint32_t rw[DROP ? 16 : 1];
        if constexpr (DROP) {
          const uint32_t bh = (uint32_t)(U.b * p.H + U.h), kg = (uint32_t)key >> 2;
          const uint32_t g0 = (uint32_t)i0 / 4u + (uint32_t)(lane & 3);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint4 r4 = philox4x32_10(kg, g0 + 4u * m, bh, p.drop.offset, p.drop.seed_lo, p.drop.seed_hi);
            const uint32_t a0 = prmt(r4.x, r4.y, 0x5140u), a1 = prmt(r4.x, r4.y, 0x7362u);
            const uint32_t a2 = prmt(r4.z, r4.w, 0x5140u), a3 = prmt(r4.z, r4.w, 0x7362u);
            uint32_t x[4] = {prmt(a0, a2, 0x5410u), prmt(a0, a2, 0x7632u), prmt(a1, a3, 0x5410u),
                             prmt(a1, a3, 0x7632u)};
            quad_transpose(x, lane);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) rw[4 * m + c4] = x[c4];
          }
        }
        // ---- Pᵀ = 2^(c·Sᵀ − LSE·log2 e), masked
        if (!warp_wait_b(bar(C::B_SFULL), g & 1, wd)) { ok = false; break; }
        tc_fence_after();
        // Pᵀ is kept in registers only in its packed 16-bit form (the values the dV product uses), which
        // leaves registers for the dQ warpgroup to take its whole partial out of tensor memory at once
        uint32_t pk[32];
        {
          uint32_t sr[64];
          tmem_ld64(tS, sr);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(C::B_SREAD));
          float pt[64];
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), c2,
                                        make_float2(lse_h[i], lse_h[i + 1]));
            if (((DROP ? 0u : BwdPolyMask<D>::value) >> ((i >> 1) & 7)) & 1u) {  // dropout: registers are short
              const float2 e = exp2_poly2(x);
              pt[i] = e.x;
              pt[i + 1] = e.y;
            } else {
              pt[i] = ex2(x.x);
              pt[i + 1] = ex2(x.y);
            }
          }
          if (!full) {
#pragma unroll
            for (int i = 0; i < 64; ++i) pt[i] = (i >= q_lo && i < q_hi) ? pt[i] : 0.f;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = pack2<BF16>(pt[2 * i], pt[2 * i + 1]);
        }
        // packed over [32a, 32a + 32): for a = 1 those are Sᵀ columns of half 0, so both halves must have
        // been read first (half 0 packs over its own columns), and at d = 128 dQᵀ of the previous step
        // (written over Sᵀ after that) must have been read out
        if ((a == 1 && !warp_wait_b(bar(C::B_SREAD), g & 1, wd)) ||
            (!C::DQ_OWN && g > 0 && !warp_wait_b(bar(C::B_DQFREE), (g - 1) & 1, wd))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if constexpr (DROP) {
          // the dV product takes the dropped Pᵀ (its 1/(1 − p) is applied to dV at the end); pk keeps
          // the undropped values for dSᵀ
#pragma unroll
          for (int hq = 0; hq < 2; ++hq) {
            uint32_t pd[16];
#pragma unroll
            for (int w = 0; w < 8; ++w) {  // word w of this 32-query quarter: pairs 2w, 2w + 1
              uint32_t m01, m23;
              keep_pair_masks(rw[8 * hq + w], keep_bias, m01, m23);
              pd[2 * w] = pk[16 * hq + 2 * w] & m01;
              pd[2 * w + 1] = pk[16 * hq + 2 * w + 1] & m23;
            }
            tmem_st16(tP + 16u * hq, pd);
          }
        } else {
          tmem_st32(tP, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_PREADY + a));
        // ---- dSᵀ = Pᵀ ∘ (dPᵀ − D)
        if (!warp_wait_b(bar(C::B_DPFULL), g & 1, wd)) { ok = false; break; }
        tc_fence_after();
        uint32_t dsk[32];
        {
          uint32_t dr[64];
          tmem_ld64(tDP, dr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 dpv = make_float2(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1]));
            float2 dd;
            if constexpr (DROP) {
              // dSᵀ = Pᵀ ∘ (Z ∘ dPᵀ / (1 − p) − D): the keep flag's sign fills the factor's 32 bits
              uint32_t e, o;
              keep_flags(rw[i >> 1], keep_bias, e, o);  // once per word: the compiler shares it across i, i ^ 1
              const float f0 = __uint_as_float(prmt(e, o, (i & 1) ? 0xBBBBu : 0x9999u) & ks_bits);
              const float f1 = __uint_as_float(prmt(e, o, (i & 1) ? 0xFFFFu : 0xDDDDu) & ks_bits);
              dd = __ffma2_rn(dpv, make_float2(f0, f1), make_float2(del_h[2 * i], del_h[2 * i + 1]));
            } else {
              dd = __fadd2_rn(dpv, make_float2(del_h[2 * i], del_h[2 * i + 1]));
            }
            const float2 ds = __fmul2_rn(unpack2<BF16>(pk[i]), dd);
            dsk[i] = pack2<BF16>(ds.x, ds.y);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(C::B_DPREAD));
        // into shared-memory chunk a as a 128-byte swizzled row (B operand of dQᵀ)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(ds_row + ((j ^ (kr & 7)) << 4)) =
              make_uint4(dsk[4 * j], dsk[4 * j + 1], dsk[4 * j + 2], dsk[4 * j + 3]);
        fence_proxy_async_smem();
        // packed over [128 + 32a, ...) (A operand of dK): for a = 1 those are dPᵀ columns of half 0, so both
        // halves must have been read first (half 0 packs over its own columns)
        if (a == 1 && !warp_wait_b(bar(C::B_DPREAD), g & 1, wd)) { ok = false; break; }
        tc_fence_after();
        tmem_st32(tDS, dsk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_DSREADY + a));
      }
    }
    __syncwarp();
  } else {
    // ================================================================ dQ warpgroup (warps 8-11)
    // Per step, thread = feature of the dQ partial; per unit, thread = key row of the dK and dV epilogue.
    regs_set<C::REGS_DQ, C::REGS_LAUNCH>();
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t tDQ = tmem + lane_off + C::T_DQ;
    const uint32_t tDK = tmem + lane_off + C::T_DK;
    const uint32_t tDV = tmem + lane_off + C::T_DV;
    // this warp's two staging boxes: row q = query, 32 fp32 features in 16-byte chunks swizzled by q mod 8
    const uint32_t box_base = s_base + C::OFF_DQS + quarter * 2 * C::DQ_BOX;
    uint32_t g = 0;       // steps so far (all units)
    uint32_t u = 0;       // units so far
    uint32_t pieces = 0;  // boxes staged so far (box = pieces mod 2)
    bool ok = true;
    int unit;
    while (ok && read_unit(unit) && unit >= 0) {
      BwdUnit U;
      decode_bwd_unit(p, unit, U, false);
      for (int it = 0; it < U.n_it; ++it, ++g) {
        const int i0 = (U.i_begin + it) * BQ;
        if (!warp_wait_b(bar(C::B_DQFULL), g & 1, wd)) { ok = false; break; }
        tc_fence_after();
        if constexpr (!C::DQ_OWN) {
          // dQᵀ: the whole partial into registers (lane = feature 32·quarter + lane, columns = queries), so
          // that [0, 128) is released at once; staging and the reduce-adds follow at their own pace
          uint32_t qr[128];
          tmem_ld64(tDQ, reinterpret_cast<uint32_t(&)[64]>(qr[0]));
          tmem_ld64(tDQ + 64u, reinterpret_cast<uint32_t(&)[64]>(qr[64]));
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(C::B_DQFREE));
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int q0 = i0 + 32 * c;
            if (q0 >= U.L) break;  // the rest of the step lies past the sequence: nothing to add
            const uint32_t bx = box_base + (pieces & 1u) * C::DQ_BOX;
            // the box may be rewritten once the reduce issued from it two pieces ago has read it
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 32; ++q)
              st_shared_f32(bx + q * 128 + (((lane >> 2) ^ (q & 7)) << 4) + ((lane & 3) << 2), qr[32 * c + q]);
            fence_proxy_async_smem();
            __syncwarp();
            // rows past the sequence hold exact zeros (P is 0 there); rows past T are clipped by the TMA unit
            if (lane == 0) {
              tma_reduce_add_3d(&tm_dq, bx, 32 * quarter, U.h, U.tok0 + q0);
              bulk_commit_group();
            }
            __syncwarp();
            ++pieces;
          }
        } else {
          // dQ: lane = query 32·quarter + lane of the step, columns = the 64 features; this warp's 32 query
          // rows go out as two boxes of 32 features
          uint32_t qr[64];
          tmem_ld64(tDQ, qr);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(C::B_DQFREE));
          const int q0 = i0 + 32 * quarter;
          if (q0 < U.L) {
            // both boxes may be rewritten once the reduces issued from them last step have read them
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
#pragma unroll
            for (int bx_i = 0; bx_i < 2; ++bx_i) {
              const uint32_t row = box_base + bx_i * C::DQ_BOX + lane * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                st_shared_v4(row + ((j ^ (lane & 7)) << 4), qr[32 * bx_i + 4 * j], qr[32 * bx_i + 4 * j + 1],
                             qr[32 * bx_i + 4 * j + 2], qr[32 * bx_i + 4 * j + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            // rows past the sequence hold exact zeros (P is 0 there); rows past T are clipped by the TMA unit
            if (lane == 0) {
              tma_reduce_add_3d(&tm_dq, box_base, 0, U.h, U.tok0 + q0);
              tma_reduce_add_3d(&tm_dq, box_base + C::DQ_BOX, 32, U.h, U.tok0 + q0);
              bulk_commit_group();
            }
            __syncwarp();
          }
        }
      }
      if (!ok) break;
      // ---- epilogue of the unit: dK (× scale) and dV rows of the key tile, read out of tensor memory
      // (released to the next unit's first products as soon as they are in registers) and stored
      if (!warp_wait_b(bar(C::B_DKV), u & 1, wd)) { ok = false; break; }
      tc_fence_after();
      const int key = U.k0 + 32 * quarter + lane;
      const bool valid = key < U.L;
      uint8_t* dk_row = reinterpret_cast<uint8_t*>(p.dk) + (((size_t)(U.tok0 + (valid ? key : 0)) * p.H + U.h) * D) * 2;
      uint8_t* dv_row = reinterpret_cast<uint8_t*>(p.dv) + (((size_t)(U.tok0 + (valid ? key : 0)) * p.H + U.h) * D) * 2;
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {  // dK, then dV
        const float f = t == 0 ? p.scale : (DROP ? p.drop.keep_scale : 1.f);  // dV: the dropout's 1/(1 − p)
        uint8_t* row = t == 0 ? dk_row : dv_row;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t r32[32];
          tmem_ld32((t == 0 ? tDK : tDV) + 32u * q, r32);
          tmem_wait_ld();
          if (t == 1 && q == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar(C::B_DKVFREE));  // dK and dV read out: the next unit may overwrite them
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2<BF16>(__uint_as_float(r32[2 * i]) * f, __uint_as_float(r32[2 * i + 1]) * f);
          if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              st_global_v4(row + q * 64 + v4 * 16, pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
      }
      ++u;
    }
    if (lane == 0) bulk_wait_group_all();  // every reduce performed before the kernel ends
    __syncwarp();
  }

  // ---- tear-down
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================================ launchers

static int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int D, bool BF16>
static cudaError_t launch_pre_t(const Problem& pb, const BwdArgs& a, cudaStream_t stream) {
  const long long rows = (long long)pb.T * pb.H;
  const long long threads = rows * (D / 8);
  long long blocks = (threads + 255) / 256;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  fa_bwd_pre_kernel<D, BF16><<<(unsigned)blocks, 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(a.o), reinterpret_cast<const uint4*>(a.dO), a.delta,
      reinterpret_cast<float4*>(a.dq_acc), rows);
  return cudaPeekAtLastError();
}

cudaError_t launch_bwd_pre(const Problem& pb, const BwdArgs& a, cudaStream_t stream) {
  if (pb.d == 128) return pb.bf16 ? launch_pre_t<128, true>(pb, a, stream) : launch_pre_t<128, false>(pb, a, stream);
  return pb.bf16 ? launch_pre_t<64, true>(pb, a, stream) : launch_pre_t<64, false>(pb, a, stream);
}

cudaError_t launch_bwd_post(const Problem& pb, const BwdArgs& a, cudaStream_t stream) {
  const long long n4 = (long long)pb.T * pb.H * pb.d / 4;
  long long blocks = (n4 + 255) / 256;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  const long long row4 = (long long)pb.H * pb.d / 4;
  if (pb.bf16)
    fa_bwd_post_kernel<true><<<(unsigned)blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(a.dq_acc),
                                                                   reinterpret_cast<uint2*>(a.dq), n4, pb.scale,
                                                                   pb.cu_seqlens, pb.B, row4);
  else
    fa_bwd_post_kernel<false><<<(unsigned)blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(a.dq_acc),
                                                                    reinterpret_cast<uint2*>(a.dq), n4, pb.scale,
                                                                    pb.cu_seqlens, pb.B, row4);
  return cudaPeekAtLastError();
}

template <int D, bool BF16, bool DROP>
static cudaError_t launch_main_q128_t(const Problem& pb, const BwdArgs& a, cudaStream_t stream) {
  static std::atomic<unsigned long long> configured{0};  // per instantiation, one bit per device
  auto kern = fa_bwd_main_q128_kernel<D, BF16, DROP>;
  if (cudaError_t e = set_smem_once(configured, reinterpret_cast<const void*>(kern), Bq128<D>::SMEM_BYTES);
      e != cudaSuccess)
    return e;
  BwdParams p;
  p.lse = a.lse;
  p.delta = a.delta;
  p.dq_acc = a.dq_acc;
  p.dk = a.dk;
  p.dv = a.dv;
  p.cu_seqlens = pb.cu_seqlens;
  p.B = pb.B;
  p.H = pb.H;
  p.N = pb.N;
  p.T = pb.T;
  p.causal = pb.causal;
  p.num_kblocks = (pb.N + kBK - 1) / kBK;
  p.heads_group = 8;
  p.scale = pb.scale;
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.timeout_ns = pb.timeout_ns;
  p.drop = pb.drop;
  const long long units = (long long)pb.B * pb.H * p.num_kblocks;
  kern<<<dim3((unsigned)units), dim3(kBwd128Threads), Bq128<D>::SMEM_BYTES, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_do,
                                                                                     a.tm_dq, p);
  return cudaPeekAtLastError();
}

template <bool DROP>
static cudaError_t launch_main_d(const Problem& pb, const BwdArgs& a, cudaStream_t stream) {
  if (pb.d == 128)
    return pb.bf16 ? launch_main_q128_t<128, true, DROP>(pb, a, stream)
                   : launch_main_q128_t<128, false, DROP>(pb, a, stream);
  return pb.bf16 ? launch_main_q128_t<64, true, DROP>(pb, a, stream) : launch_main_q128_t<64, false, DROP>(pb, a, stream);
}

// Rows per Q / dO tile the main kernel loads, and per box of its dQ reduce-adds (the host encodes the
// tensor maps with these box heights).
int bwd_q_tile_rows(int, bool) { return 128; }
int bwd_dq_box_rows(int, bool) { return 32; }

cudaError_t launch_bwd_main(const Problem& pb, const BwdArgs& a, cudaStream_t stream) {
  return pb.drop.t != 0u ? launch_main_d<true>(pb, a, stream) : launch_main_d<false>(pb, a, stream);
}

// ============================================================================ watchdog self-test

__global__ void fa_watchdog_selftest_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t never;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&never), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const Watchdog wd{&abort_flag, timeout_ns};
  // nothing arrives on `never`: the wait must give up and record FA_ERR_TIMEOUT
  mbar_wait(smem_u32(&never), 0, wd);
  __syncthreads();
}

cudaError_t launch_watchdog_selftest(uint64_t timeout_ns, cudaStream_t stream) {
  fa_watchdog_selftest_kernel<<<1, 64, 0, stream>>>(timeout_ns);
  return cudaPeekAtLastError();
}

}  // namespace fa
