// fa_fwd.cu — attention forward for sm_100a.
//
// Computes O = softmax(Q Kᵀ·scale [+ causal mask]) V and the row log-sum-exp
// tile by tile with an online softmax ("FlashAttention 详解（零基础入门）" §5.2,
// §5.4, §6.2): the [128 × 128] score tile S lives only in tensor memory, P is
// written back over it in the input dtype and fed to the P·V MMA from there,
// so neither S nor P ever reaches device memory.
//
// CTA = one work unit = (sequence, head, 256 query rows) split into two
// 128-row Q tiles that take turns on the tensor core:
//   warps 0-3  softmax of Q tile 0 (one thread per row; TMEM lanes 0-127)
//   warps 4-7  softmax of Q tile 1
//   warp  8    TMA producer: Q0/Q1 once, then the K and V rings
//   warp  9    tensor-memory allocator and MMA issuer (one elected lane)
//   warps 10-11 idle (they complete the third warpgroup, whose registers
//              setmaxnreg hands to the softmax warpgroups: 208 / 208 / 88)
// K_j and V_j have separate empty barriers: K_j's stage is handed back to
// the producer as soon as both S(·, j) products are done, so the next K tile
// streams in while P·V(·, j) still reads V_j.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d),
// O1 [256+d, 256+2d).  MMA issue order per KV tile j:
//   P·V(0,j)  S(0,j+1)  P·V(1,j)  S(1,j+1)
// so while one warpgroup exponentiates, the tensor core works for the other.
// tcgen05 MMAs from one thread execute in issue order, so S(t,j+1) may
// overwrite the columns holding P(t,j) once P·V(t,j) has been issued.
//
// Online softmax in base 2 with c = scale·log2(e): m is kept in the scaled
// domain and P = 2^(c·s − m).  The running max is only raised when the tile
// max exceeds it by more than 8 (a factor 256): O and ℓ are then both
// expressed against the same, slightly stale reference, which leaves
// O = Σ P V / Σ P unchanged (the rescaling argument of §5.2 run in reverse),
// keeps every P ≤ 256, and makes the O rescale in tensor memory rare.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

struct FwdParams {
  void* o;
  float* lse;
  const int32_t* cu_seqlens;
  int B, H, N, T;
  int causal;
  int num_qblocks;   // ceil(N / 256)
  int heads_group;   // heads per L2 group in the unit order
  float scale_log2;  // scale · log2(e)
  uint64_t timeout_ns;
};

constexpr int kFwdThreads = 384;  // 3 warpgroups
constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr float kRescaleThreshold = 8.0f;
// Column pairs i (of 64 per row) with bit (i % 8) set take the FMA-pipe exp2 in unmasked tiles.  At
// d = 128 the tensor core needs as long per tile as the MUFU, and the polynomial costs about as much
// per element as ex2, so it stays off; at d = 64 the MMAs take half as long and the exponentials bound
// the tile, so part of them moves to the FMA pipe.
template <int D> struct PolyMask { static constexpr uint32_t value = 0x00u; };
template <> struct PolyMask<64> { static constexpr uint32_t value = 0x22u; };

template <int D>
struct FwdCfg {
  static constexpr int NCH = D / 64;                   // 128-byte feature chunks per row
  static constexpr uint32_t TILE = kBM * D * 2;        // bytes of a 128-row tile
  static constexpr int KSTAGES = (D == 128) ? 3 : 5;   // K ring depth
  static constexpr int VSTAGES = (D == 128) ? 2 : 4;   // V ring depth
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + KSTAGES;
  static constexpr int B_VFULL = B_KEMPTY + KSTAGES;
  static constexpr int B_VEMPTY = B_VFULL + VSTAGES;
  static constexpr int B_SFULL = B_VEMPTY + VSTAGES;
  static constexpr int B_PFULL = B_SFULL + 2;
  static constexpr int B_PVDONE = B_PFULL + 2;
  static constexpr int B_DRAIN = B_PVDONE + 2;
  static constexpr int NBARS = B_DRAIN + 1;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = 2 * TILE;
  static constexpr uint32_t OFF_V = OFF_K + KSTAGES * TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + VSTAGES * TILE;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Bounded wait that ignores the abort flag: used on the way out, for work
// that completes on its own (outstanding TMA loads and MMAs).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      record_status(4);
      return;
    }
  }
}

// Warp-uniform bounded wait: every lane waits, and the warp proceeds only if
// all lanes succeeded (keeps the .sync.aligned tensor-memory instructions that
// follow convergent even when one lane's wait gives up).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Watchdog& wd) {
  const bool ok = mbar_wait(bar, parity, wd);
  return __all_sync(0xffffffffu, ok);
}

// S = Q·Kᵀ for one 128 × 128 tile: D/16 MMAs of K = 16 along the head dimension.
// Q and K are K-major with 128-byte rows; a 16-element step is +32 bytes inside a
// swizzle atom, a 64-element step the next 16 KB atom column.
template <int D, uint32_t IDESC>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint64_t dq, uint64_t dk) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * (kBM * 128) + (kk & 3) * 32) >> 4;
    mma_ss(s_tmem, dq + off, dk + off, IDESC, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P·V for one tile: 8 MMAs of K = 16 keys; P is read from tensor memory
// (8 columns of packed 16-bit values per step), V is MN-major (+2 KB per 16 keys).
template <uint32_t IDESC>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t dv, uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk)
    mma_ts(o_tmem, p_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), IDESC, kk > 0 ? 1u : acc);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  constexpr uint32_t IDESC_S = idesc_f16(BF16, kBM, kBN, false, false);  // S = Q·Kᵀ, both K-major
  constexpr uint32_t IDESC_O = idesc_f16(BF16, kBM, D, false, true);     // O += P·V, V MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t sQ = s_base + C::OFF_Q;
  const uint32_t sK = s_base + C::OFF_K;
  const uint32_t sV = s_base + C::OFF_V;
  const uint32_t bar0 = s_base + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- decode the work unit: heads in groups (K/V of a group stay in L2),
  //      heaviest query blocks first inside a group (causal load balance)
  const int BH = p.B * p.H;
  const int nqb = p.num_qblocks;
  const int G = p.heads_group;
  const int unit = blockIdx.x;
  const int group = unit / (G * nqb);
  const int g_heads = min(G, BH - group * G);
  const int r = unit - group * G * nqb;
  const int qb = nqb - 1 - r / g_heads;
  const int bh = group * G + r % g_heads;
  const int b = bh / p.H;
  const int h = bh - b * p.H;

  int tok0, L;
  if (p.cu_seqlens != nullptr) {
    tok0 = __ldg(p.cu_seqlens + b);
    const int end = __ldg(p.cu_seqlens + b + 1);
    L = end - tok0;
    if (tok0 < 0 || L < 0 || end > p.T || L > p.N) {
      if (threadIdx.x == 0) record_status(1);
      return;
    }
  } else {
    tok0 = b * p.N;
    L = p.N;
  }
  const int q0 = qb * 2 * kBM;
  if (q0 >= L) return;  // uniform over the CTA: nothing allocated yet
  const int nkv_all = (L + kBN - 1) / kBN;
  int nkv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int first_row = q0 + t * kBM;
    if (first_row >= L) nkv[t] = 0;
    else nkv[t] = p.causal ? min(nkv_all, (first_row + kBM - 1) / kBN + 1) : nkv_all;
  }
  const int n_iter = max(nkv[0], nkv[1]);

  // ---- set-up: barriers, tensor memory
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::KSTAGES; ++s) {
      mbar_init(bar(C::B_KFULL + s), 1);
      mbar_init(bar(C::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < C::VSTAGES; ++s) {
      mbar_init(bar(C::B_VFULL + s), 1);
      mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::B_SFULL + t), 1);
      mbar_init(bar(C::B_PFULL + t), kBM);
      mbar_init(bar(C::B_PVDONE + t), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, p.timeout_ns};

  if (warp >= 8) {
    regs_dec<88>();
    // The producer and MMA warps run their loops with all 32 lanes (warp-uniform state the
    // compiler can keep in uniform registers); one elected lane issues each TMA copy, MMA and
    // commit.  elect.sync picks the lowest active lane, so every MMA and every commit that
    // tracks it come from the same thread.
    if (warp == 8) {
      // ================================================================ TMA producer
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      const int nq = nkv[1] > 0 ? 2 : 1;
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(C::B_Q), nq * C::TILE);
        for (int t = 0; t < nq; ++t)
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(sQ + t * C::TILE + c * (kBM * 128), &tm_q, bar(C::B_Q), c * 64, h, tok0 + q0 + t * kBM,
                        pol_q);
      }
      __syncwarp();
      int issued = 0;
      for (int j = 0; j < n_iter; ++j) {
        const int sk = j % C::KSTAGES, sv = j % C::VSTAGES;
        if (j >= C::KSTAGES && !warp_wait(bar(C::B_KEMPTY + sk), ((j / C::KSTAGES) - 1) & 1, wd)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(C::B_KFULL + sk), C::TILE);
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(sK + sk * C::TILE + c * (kBN * 128), &tm_k, bar(C::B_KFULL + sk), c * 64, h, tok0 + j * kBN,
                        pol_kv);
        }
        __syncwarp();
        if (j >= C::VSTAGES && !warp_wait(bar(C::B_VEMPTY + sv), ((j / C::VSTAGES) - 1) & 1, wd)) {
          issued = -(j + 1);  // K_j issued, V_j not
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(C::B_VFULL + sv), C::TILE);
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(sV + sv * C::TILE + c * (kBN * 128), &tm_v, bar(C::B_VFULL + sv), c * 64, h, tok0 + j * kBN,
                        pol_kv);
        }
        __syncwarp();
        issued = j + 1;
      }
      // Let every load this warp issued land before the CTA can exit.
      if (elect_one()) {
        const int k_issued = issued >= 0 ? issued : -issued;
        const int v_issued = issued >= 0 ? issued : -issued - 1;
        drain_wait(bar(C::B_Q), 0, p.timeout_ns);
        for (int j = max(0, k_issued - C::KSTAGES); j < k_issued; ++j)
          drain_wait(bar(C::B_KFULL + j % C::KSTAGES), (j / C::KSTAGES) & 1, p.timeout_ns);
        for (int j = max(0, v_issued - C::VSTAGES); j < v_issued; ++j)
          drain_wait(bar(C::B_VFULL + j % C::VSTAGES), (j / C::VSTAGES) & 1, p.timeout_ns);
      }
      __syncwarp();
    } else if (warp == 9) {
      // ================================================================ MMA issuer
      // Descriptors are computed once; per instruction only a constant start-address offset
      // (in 16-byte units, no carry out of the 14-bit field: shared addresses stay below 228 KB).
      const uint64_t dq_base = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk_base = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv_base = sdesc_sw128(sV, kBN * 128, 1024);
      bool ok = warp_wait(bar(C::B_Q), 0, wd) && warp_wait(bar(C::B_KFULL + 0), 0, wd);
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          if (nkv[0] > 0) {
            issue_qk<D, IDESC_S>(tmem + 0u, dq_base, dk_base);
            tc_commit(bar(C::B_SFULL + 0));
          }
          if (nkv[1] > 0) {
            issue_qk<D, IDESC_S>(tmem + 128u, dq_base + (C::TILE >> 4), dk_base);
            tc_commit(bar(C::B_SFULL + 1));
          }
          tc_commit(bar(C::B_KEMPTY + 0));  // K_0 is read by no later MMA
        }
        __syncwarp();
      }
      for (int j = 0; ok && j < n_iter; ++j) {
        const int s = j % C::VSTAGES;                  // V_j
        const uint32_t ph = (j / C::VSTAGES) & 1;
        const uint64_t dv_s = dv_base + ((s * C::TILE) >> 4);
        const int s1 = (j + 1) % C::KSTAGES;           // K_{j+1}
        const uint64_t dk_s1 = dk_base + ((s1 * C::TILE) >> 4);
        bool v_ready = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (j >= nkv[t]) continue;
          const uint32_t s_tmem = tmem + 128u * t;
          const uint32_t o_tmem = tmem + 256u + (uint32_t)D * t;
          if (!warp_wait(bar(C::B_PFULL + t), j & 1, wd)) { ok = false; break; }
          if (!v_ready) {
            if (!warp_wait(bar(C::B_VFULL + s), ph, wd)) { ok = false; break; }
            v_ready = true;
          }
          tc_fence_after();
          if (elect_one()) {
            issue_pv<IDESC_O>(o_tmem, s_tmem, dv_s, j > 0 ? 1u : 0u);
            if (nkv[t] == 1) issue_pv<IDESC_O>(o_tmem, s_tmem + 64u, dv_s, 1u);  // lo part of a split P
            tc_commit(bar(C::B_PVDONE + t));
          }
          __syncwarp();
          if (j + 1 < nkv[t]) {
            if (!warp_wait(bar(C::B_KFULL + s1), ((j + 1) / C::KSTAGES) & 1, wd)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              issue_qk<D, IDESC_S>(s_tmem, dq_base + ((t * C::TILE) >> 4), dk_s1);
              tc_commit(bar(C::B_SFULL + t));
            }
            __syncwarp();
          }
        }
        if (elect_one()) {
          tc_commit(bar(C::B_VEMPTY + s));                     // V_j: both P·V(·, j) issued
          if (j + 1 < n_iter) tc_commit(bar(C::B_KEMPTY + s1));  // K_{j+1}: both S(·, j+1) issued
        }
        __syncwarp();
      }
      // every MMA issued so far must finish before tensor memory is released
      if (elect_one()) {
        tc_commit(bar(C::B_DRAIN));
        drain_wait(bar(C::B_DRAIN), 0, p.timeout_ns);
      }
      __syncwarp();
    }
    __syncwarp();
  } else {
    // ================================================================ softmax warpgroups
    regs_inc<208>();
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int my_nkv = (t == 0) ? nkv[0] : nkv[1];
    if (my_nkv > 0) {
      const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
      const uint32_t tS = tmem + lane_off + 128u * t;
      const uint32_t tO = tmem + lane_off + 256u + (uint32_t)(D * t);
      const int row = q0 + t * kBM + 32 * quarter + lane;  // position in the sequence
      const int key_limit = p.causal ? min(L, row + 1) : L;
      const float c = p.scale_log2;
      const float2 c2 = make_float2(c, c);
      // A tile whose rows see a single KV tile (the first 128 rows of a causal
      // sequence, or a sequence of at most 128 tokens) averages few values, so
      // the rounding of P to 16 bits would show in O: there P is carried as
      // hi + lo parts and multiplied by V twice.
      const bool split_p = (my_nkv == 1);
      float m_ref = -INFINITY;  // running (possibly stale) max, scaled domain
      float ell = 0.f;
      bool ok = true;
      for (int j = 0; j < my_nkv; ++j) {
        if (!warp_wait(bar(C::B_SFULL + t), j & 1, wd)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[kBN];
#pragma unroll
        for (int q = 0; q < kBN / 32; ++q) tmem_ld32(tS + 32u * q, reinterpret_cast<uint32_t(&)[32]>(sr[32 * q]));
        tmem_wait_ld();
        float sv[kBN];
#pragma unroll
        for (int i = 0; i < kBN; ++i) sv[i] = __uint_as_float(sr[i]);
        const int lim = key_limit - j * kBN;  // keys [lim, 128) of this tile are hidden from this row
        const bool need_mask = __any_sync(0xffffffffu, lim < kBN);  // warp-uniform
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < kBN; ++i) sv[i] = (i < lim) ? sv[i] : -INFINITY;
        }
        // row max: 8 independent chains of 3-input max, then a short tree
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(sv[k], sv[k + 8]);
#pragma unroll
        for (int i = 16; i < kBN; i += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = max3f(mx[k], sv[i + k], sv[i + k + 8]);
        }
        const float m_tile = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * c;
        // raise the reference max only when the tile max exceeds it by more than the threshold
        const float m_new = (m_tile > m_ref + kRescaleThreshold) ? m_tile : m_ref;
        const float alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
        const bool rescale_o = (j > 0) && (m_new != m_ref);
        ell *= alpha;
        m_ref = m_new;
        // a row that has seen no visible key yet keeps m = -inf; its P is 0 either way
        const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if (!split_p && !need_mask && PolyMask<D>::value != 0u) {
          // unmasked tile: part of the exponentials on the FMA pipe, interleaved with the MUFU ones
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int idx = 64 * q + 2 * i;
              const float2 x = __ffma2_rn(make_float2(sv[idx], sv[idx + 1]), c2, nm2);
              float2 e;
              if ((PolyMask<D>::value >> (i & 7)) & 1u) e = exp2_poly2(x);
              else e = make_float2(ex2(x.x), ex2(x.y));
              acc[i & 3] = __fadd2_rn(acc[i & 3], e);
              pk[i] = pack2<BF16>(e.x, e.y);
            }
            tmem_st32(tS + 32u * q, pk);
          }
        } else if (!split_p) {
          // P = 2^(c·s − m) on the MUFU (ex2(−inf) = 0 exactly), packed to 16 bits, written over S
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int idx = 64 * q + 2 * i;
              const float2 x = __ffma2_rn(make_float2(sv[idx], sv[idx + 1]), c2, nm2);
              const float2 e = make_float2(ex2(x.x), ex2(x.y));
              acc[i & 3] = __fadd2_rn(acc[i & 3], e);
              pk[i] = pack2<BF16>(e.x, e.y);
            }
            tmem_st32(tS + 32u * q, pk);
          }
        } else {
          // P = hi + lo, both in the input dtype: hi in columns [0, 64), lo in [64, 128)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int idx = 32 * q + 2 * i;
              const float2 x = __ffma2_rn(make_float2(sv[idx], sv[idx + 1]), c2, nm2);
              const float2 e = make_float2(ex2(x.x), ex2(x.y));
              acc[i & 3] = __fadd2_rn(acc[i & 3], e);
              hi[i] = pack2<BF16>(e.x, e.y);
              const float2 hf = unpack2<BF16>(hi[i]);
              lo[i] = pack2<BF16>(e.x - hf.x, e.y - hf.y);
            }
            tmem_st16(tS + 16u * q, hi);
            tmem_st16(tS + 64u + 16u * q, lo);
          }
        }
        const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        ell += a.x + a.y;
        if (__any_sync(0xffffffffu, rescale_o)) {
          // The reference max rose (rare past the first tile): O(t) must hold P·V(t, j-1) before it
          // is rescaled, and the rescale must land before P·V(t, j) is issued.
          if (!warp_wait(bar(C::B_PVDONE + t), (j - 1) & 1, wd)) { ok = false; break; }
          tc_fence_after();
          const float f = rescale_o ? alpha : 1.f;
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t r32[32];
            tmem_ld32(tO + 32u * q, r32);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(__uint_as_float(r32[i]) * f);
            tmem_st32(tO + 32u * q, r32);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + t));
      }
      // ---- epilogue: O / ℓ -> dtype, LSE
      if (ok && warp_wait(bar(C::B_PVDONE + t), (my_nkv - 1) & 1, wd)) {
        tc_fence_after();
        const bool valid = row < L;
        const float inv = (ell > 0.f) ? 1.f / ell : 0.f;
        const size_t obase = ((size_t)(tok0 + (valid ? row : 0)) * p.H + h) * D;
        uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) + obase * 2;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t r32[32];
          tmem_ld32(tO + 32u * q, r32);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2<BF16>(__uint_as_float(r32[2 * i]) * inv, __uint_as_float(r32[2 * i + 1]) * inv);
          if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              st_global_v4(orow + q * 64 + v4 * 16, pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
        if (valid) {
          const float lse = (ell > 0.f && m_ref != -INFINITY) ? (m_ref + __log2f(ell)) * 0.69314718055994531f
                                                             : -INFINITY;
          p.lse[(size_t)(tok0 + row) * p.H + h] = lse;
        }
      }
    }
    __syncwarp();
  }

  // ---- tear-down
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool BF16>
static cudaError_t launch_fwd_t(const Problem& pb, const FwdArgs& a, cudaStream_t stream) {
  using C = FwdCfg<D>;
  static bool configured = false;  // per instantiation
  auto kern = fa_fwd_kernel<D, BF16>;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  FwdParams p;
  p.o = a.o;
  p.lse = a.lse;
  p.cu_seqlens = pb.cu_seqlens;
  p.B = pb.B;
  p.H = pb.H;
  p.N = pb.N;
  p.T = pb.T;
  p.causal = pb.causal;
  p.num_qblocks = (pb.N + 2 * kBM - 1) / (2 * kBM);
  p.heads_group = 8;
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.timeout_ns = pb.timeout_ns;
  const long long units = (long long)pb.B * pb.H * p.num_qblocks;
  kern<<<dim3((unsigned)units), dim3(kFwdThreads), C::SMEM_BYTES, stream>>>(a.tm_q, a.tm_k, a.tm_v, p);
  return cudaPeekAtLastError();
}

cudaError_t launch_fwd(const Problem& pb, const FwdArgs& a, cudaStream_t stream) {
  if (pb.d == 128) return pb.bf16 ? launch_fwd_t<128, true>(pb, a, stream) : launch_fwd_t<128, false>(pb, a, stream);
  return pb.bf16 ? launch_fwd_t<64, true>(pb, a, stream) : launch_fwd_t<64, false>(pb, a, stream);
}

}  // namespace fa
