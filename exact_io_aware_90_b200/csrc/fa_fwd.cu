// fa_fwd.cu — attention forward for sm_100a.
//
// Computes O = softmax(Q Kᵀ·scale [+ causal mask]) V and the row log-sum-exp
// tile by tile with an online softmax ("FlashAttention 详解（零基础入门）" §5.2,
// §5.4, §6.2): the [128 × 128] score tile S lives only in tensor memory, P is
// written back over it in the input dtype and fed to the P·V MMA from there,
// so neither S nor P ever reaches device memory.
//
// Work unit = (sequence, head, 256 query rows), split into two 128-row Q
// tiles that take turns on the tensor core.  The kernel is persistent: the
// grid has one CTA per unit, but a running CTA keeps its tensor memory,
// barriers and pipelines and takes further units from the hardware scheduler
// (cluster launch control: it cancels the launch of a CTA that has not started
// yet and does that CTA's unit), so on a busy GPU ~one CTA per SM does all the
// work, and the next unit's first score tiles are computed while the current
// unit's last P·V and O epilogue run.
//   warps 0-3  softmax of Q tile 0 (one thread per row; TMEM lanes 0-127)
//   warps 4-7  softmax of Q tile 1
//   warp  8    scheduler and TMA producer: Q0/Q1 per unit, the K and V rings
//   warp  9    tensor-memory allocator and MMA issuer (one elected lane)
//   warps 10-11 idle (they complete the third warpgroup, whose registers
//              setmaxnreg hands to the softmax warpgroups: 200 / 200 / 104)
// K_j and V_j have separate empty barriers: K_j's stage is handed back to
// the producer as soon as both S(·, j) products are done, so the next K tile
// streams in while P·V(·, j) still reads V_j.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d),
// O1 [256+d, 256+2d).  MMA issue order per KV tile j:
//   P·V(0,j)  S(0,j+1)  P·V(1,j)  S(1,j+1)
// so while one warpgroup exponentiates, the tensor core works for the other.
// tcgen05 MMAs from one thread execute in issue order, so S(t,j+1) may
// overwrite the columns holding P(t,j) once P·V(t,j) has been issued; the
// same holds for S(t,0) of the next unit after the last P·V(t,·) of this one.
//
// Online softmax in base 2 with c = scale·log2(e): m is kept in the scaled
// domain and P = 2^(c·s − m).  The running max is only raised when the tile
// max exceeds it by more than 8 (a factor 256): O and ℓ are then both
// expressed against the same, slightly stale reference, which leaves
// O = Σ P V / Σ P unchanged (the rescaling argument of §5.2 run in reverse),
// keeps every P ≤ 256, and makes the O rescale in tensor memory rare.
//
// e4m3 inputs (the FP8 instantiation, d = 128): Q, K, V tiles are 128-byte rows of 8-bit values
// (16 KB per tile, deeper K/V rings), S and P·V run as kind::f8f6f4 MMAs of K = 32, the per-tensor
// descales of q and k are folded into c and v's multiplies O in the epilogue, P is rounded to e4m3
// (≤ 256 < 448, so no saturation) and packed four keys per tensor-memory column, and O is written
// as bf16.
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
  float scale_log2;  // scale · log2(e) (· the q and k descales for e4m3 inputs)
  float o_scale;     // factor on O at the end: 1, or the v descale for e4m3 inputs
  // e4m3 inputs with one descale per (sequence, head) (fp32 [B·H] device arrays, index b·H + h), or
  // nullptr when the descales are per tensor (folded into scale_log2 and o_scale on the host)
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
  // > 0: the descale arrays hold one value per (128-token block, head) instead, [num_blocks·H], the
  // blocks of each sequence numbered after those of the sequences before it
  int descale_blocks;
  uint64_t timeout_ns;
  Dropout drop;
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
// The e4m3 instantiation (d = 128, MMAs at twice the 16-bit rate): the same quarter, in every tile (the
// polynomial clamps its input at −126, so a masked key's 2^-126 rounds to e4m3 zero and adds nothing
// visible to ℓ).
constexpr uint32_t kFp8PolyMask = 0x22u;

// EB = bytes per input element: 2 (f16 / bf16) or 1 (e4m3).
template <int D, int EB = 2>
struct FwdCfg {
  static constexpr int NCH = D * EB / 128;             // 128-byte feature chunks per row
  static constexpr int CHUNK_ELEMS = 128 / EB;         // elements of a 128-byte chunk
  static constexpr uint32_t TILE = kBM * D * EB;       // bytes of a 128-row tile
  static constexpr int KSTAGES = (TILE == 32768) ? 3 : 5;  // K ring depth
  static constexpr int VSTAGES = (TILE == 32768) ? 2 : 4;  // V ring depth
  // barrier indices
  static constexpr int B_QFULL = 0;                   // [2] Q tile t loaded
  static constexpr int B_QEMPTY = B_QFULL + 2;        // [2] last S of Q tile t in its unit done
  static constexpr int B_KFULL = B_QEMPTY + 2;
  static constexpr int B_KEMPTY = B_KFULL + KSTAGES;
  static constexpr int B_VFULL = B_KEMPTY + KSTAGES;
  static constexpr int B_VEMPTY = B_VFULL + VSTAGES;
  static constexpr int B_SFULL = B_VEMPTY + VSTAGES;
  static constexpr int B_PFULL = B_SFULL + 2;
  static constexpr int B_PVDONE = B_PFULL + 2;
  static constexpr int B_UFULL = B_PVDONE + 2;        // [2] work-unit ring slot written
  static constexpr int B_UEMPTY = B_UFULL + 2;        // [2] slot read by the MMA warp and the 8 softmax warps
  static constexpr int B_CLC = B_UEMPTY + 2;          // scheduler response landed
  static constexpr int B_DRAIN = B_CLC + 1;
  static constexpr int NBARS = B_DRAIN + 1;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = 2 * TILE;
  static constexpr uint32_t OFF_V = OFF_K + KSTAGES * TILE;
  static constexpr uint32_t OFF_CLC = OFF_V + VSTAGES * TILE;  // 16-byte scheduler response
  static constexpr uint32_t OFF_BAR = OFF_CLC + 16;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;     // TMEM base, abort flag, unit ring [2]
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

// S = Q·Kᵀ for one 128 × 128 tile: one MMA per 32 bytes of the head dimension (K = 16
// for 16-bit inputs, 32 for e4m3).  Q and K are K-major with 128-byte rows; a 32-byte step
// stays inside a swizzle atom, the next 128 bytes are the next 16 KB atom column.
template <int D, int EB, uint32_t IDESC>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint64_t dq, uint64_t dk) {
  dq = opaque64(dq);
  dk = opaque64(dk);
#pragma unroll
  for (int kk = 0; kk < D * EB / 32; ++kk) {
    const uint32_t off = ((kk >> 2) * (kBM * 128) + (kk & 3) * 32) >> 4;
    if constexpr (EB == 1) mma_ss_f8(s_tmem, dq + off, dk + off, IDESC, kk > 0 ? 1u : 0u);
    else mma_ss(s_tmem, dq + off, dk + off, IDESC, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P·V for one tile: one MMA per 32 bytes of P's row (16 keys of 16 bits, or 32 of
// e4m3), 8 tensor-memory columns each; V is MN-major, 128 bytes per key (+2 KB per 16 keys).
template <int EB, uint32_t IDESC>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t dv, uint32_t acc) {
  dv = opaque64(dv);
  constexpr int KPM = 32 / EB;  // keys per MMA
#pragma unroll
  for (int kk = 0; kk < kBN / KPM; ++kk) {
    if constexpr (EB == 1) mma_ts_f8(o_tmem, p_tmem + kk * 8, dv + ((kk * KPM * 128) >> 4), IDESC, kk > 0 ? 1u : acc);
    else mma_ts(o_tmem, p_tmem + kk * 8, dv + ((kk * KPM * 128) >> 4), IDESC, kk > 0 ? 1u : acc);
  }
}

// A decoded work unit: query rows [q0, q0 + 256) of the sequence whose tokens
// are [tok0, tok0 + L), head h; nkv[t] KV tiles for Q tile t (0 when the tile
// lies past the end of the sequence), n_iter = max(nkv[0], nkv[1]).
struct FwdUnit {
  int tok0, L, q0, h, b;
  int nkv[2];
  int n_iter;
};

// Unit order: heads in groups (K/V of a group stay in L2), heaviest query
// blocks first inside a group (causal load balance).  Returns false for a unit
// with no query row inside its sequence; invalid sequence bounds are recorded
// as FA_ERR_INVALID_ARG and the unit is skipped.
__device__ __forceinline__ bool decode_unit(const FwdParams& p, int unit, FwdUnit& u) {
  const int BH = p.B * p.H;
  const int nqb = p.num_qblocks;
  const int G = p.heads_group;
  const int group = unit / (G * nqb);
  const int g_heads = min(G, BH - group * G);
  const int r = unit - group * G * nqb;
  const int qb = nqb - 1 - r / g_heads;
  const int bh = group * G + r % g_heads;
  const int b = bh / p.H;
  u.b = b;
  u.h = bh - b * p.H;
  if (p.cu_seqlens != nullptr) {
    u.tok0 = __ldg(p.cu_seqlens + b);
    const int end = __ldg(p.cu_seqlens + b + 1);
    u.L = end - u.tok0;
    if (u.tok0 < 0 || u.L < 0 || end > p.T || u.L > p.N) {
      record_status(1);
      return false;
    }
  } else {
    u.tok0 = b * p.N;
    u.L = p.N;
  }
  u.q0 = qb * 2 * kBM;
  if (u.q0 >= u.L) return false;
  const int nkv_all = (u.L + kBN - 1) / kBN;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int first_row = u.q0 + t * kBM;
    if (first_row >= u.L) u.nkv[t] = 0;
    else u.nkv[t] = p.causal ? min(nkv_all, (first_row + kBM - 1) / kBN + 1) : nkv_all;
  }
  u.n_iter = max(u.nkv[0], u.nkv[1]);
  return true;
}

// First per-block descale block of the unit's sequence: the ceil(L / 128) blocks of every sequence
// before it, summed across the warp (warp-collective; every lane gets the sum).
__device__ __forceinline__ int descale_block0(const FwdParams& p, const FwdUnit& u, int lane) {
  if (p.cu_seqlens == nullptr) return u.b * ((p.N + kBN - 1) / kBN);
  int n = 0;
  for (int b = lane; b < u.b; b += 32) {
    const int L = __ldg(p.cu_seqlens + b + 1) - __ldg(p.cu_seqlens + b);
    n += (max(L, 0) + kBN - 1) / kBN;
  }
  return __reduce_add_sync(0xffffffffu, n);
}

// Per-block descales: the unit's blocks must lie inside the arrays (inconsistent offsets are reported
// and the unit skipped, as decode_unit does for a bad sequence).
__device__ __forceinline__ bool descale_blocks_ok(const FwdParams& p, const FwdUnit& u, int lane) {
  if (p.descale_blocks <= 0) return true;
  const bool ok = descale_block0(p, u, lane) + (u.L + kBN - 1) / kBN <= p.descale_blocks;
  if (!ok && lane == 0) record_status(1);
  return ok;
}

// Warp-uniform non-blocking probe of one barrier phase.
__device__ __forceinline__ bool warp_test(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_test_wait(bar, parity));
}

// FP8: e4m3 Q, K, V (per-tensor descales folded into scale_log2 and o_scale), P rounded to e4m3 for
// the P·V product, O written as bf16; BF16 is then true and names the output type.
template <int D, bool BF16, bool DROP, bool FP8 = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(!(FP8 && DROP), "dropout is not built for e4m3 inputs");
  constexpr int EB = FP8 ? 1 : 2;
  using C = FwdCfg<D, EB>;
  // format code 0 is f16 for kind::f16 and e4m3 for kind::f8f6f4
  constexpr uint32_t IDESC_S = idesc_f16(BF16 && !FP8, kBM, kBN, false, false);  // S = Q·Kᵀ, both K-major
  constexpr uint32_t IDESC_O = idesc_f16(BF16 && !FP8, kBM, D, false, true);     // O += P·V, V MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t sQ = s_base + C::OFF_Q;
  const uint32_t sK = s_base + C::OFF_K;
  const uint32_t sV = s_base + C::OFF_V;
  const uint32_t clc_resp = s_base + C::OFF_CLC;
  const uint32_t bar0 = s_base + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- set-up, once per CTA: the CTA then runs work units until none is left
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::B_QFULL + t), 1);
      mbar_init(bar(C::B_QEMPTY + t), 1);
      mbar_init(bar(C::B_SFULL + t), 1);
      mbar_init(bar(C::B_PFULL + t), kBM);
      mbar_init(bar(C::B_PVDONE + t), 1);
      mbar_init(bar(C::B_UFULL + t), 1);
      mbar_init(bar(C::B_UEMPTY + t), 9);
    }
    for (int s = 0; s < C::KSTAGES; ++s) {
      mbar_init(bar(C::B_KFULL + s), 1);
      mbar_init(bar(C::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < C::VSTAGES; ++s) {
      mbar_init(bar(C::B_VFULL + s), 1);
      mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    mbar_init(bar(C::B_CLC), 1);
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
    regs_dec<104>();
    // The producer and MMA warps run their loops with all 32 lanes (warp-uniform state the
    // compiler can keep in uniform registers); one elected lane issues each TMA copy, MMA and
    // commit.  elect.sync picks the lowest active lane, so every MMA and every commit that
    // tracks it come from the same thread.
    if (warp == 8) {
      // ================================================================ scheduler and TMA producer
      // Units come from the hardware scheduler: this CTA's own index first, then, one at a time,
      // the index of a CTA of the grid that has not started yet, whose launch is cancelled.  Each
      // unit is published to the other roles through a two-slot ring.  Loads follow the order in
      // which the MMA warp consumes them across a unit boundary: Q0, K0, Q1, V0, K1, V1, ...
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      uint32_t kc = 0, vc = 0;      // K / V tiles loaded so far (ring positions)
      uint32_t qn[2] = {0u, 0u};    // loads of Q tile t
      uint32_t un = 0;              // units published
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
        if (!warp_wait(bar(C::B_CLC), c_done & 1, wd)) {
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
      auto publish = [&](int unit) -> bool {
        const int s = un & 1;
        if (un >= 2 && !warp_wait(bar(C::B_UEMPTY + s), ((un >> 1) - 1) & 1, wd)) return false;
        if (elect_one()) {
          unit_ring[s] = unit;
          mbar_arrive(bar(C::B_UFULL + s));  // release: the store is visible once the phase flips
        }
        __syncwarp();
        ++un;
        return true;
      };
      auto load_q = [&](const FwdUnit& u, int t) -> bool {
        if (qn[t] > 0 && !warp_wait(bar(C::B_QEMPTY + t), (qn[t] - 1) & 1, wd)) return false;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(C::B_QFULL + t), C::TILE);
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(sQ + t * C::TILE + c * (kBM * 128), &tm_q, bar(C::B_QFULL + t), c * C::CHUNK_ELEMS, u.h,
                        u.tok0 + u.q0 + t * kBM, pol_q);
        }
        __syncwarp();
        ++qn[t];
        return true;
      };
      auto load_k = [&](const FwdUnit& u, int j) -> bool {
        const uint32_t s = kc % C::KSTAGES;
        if (kc >= (uint32_t)C::KSTAGES && !warp_wait(bar(C::B_KEMPTY + s), ((kc / C::KSTAGES) - 1) & 1, wd))
          return false;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::TILE);
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(sK + s * C::TILE + c * (kBN * 128), &tm_k, bar(C::B_KFULL + s), c * C::CHUNK_ELEMS, u.h,
                        u.tok0 + j * kBN, pol_kv);
        }
        __syncwarp();
        ++kc;
        return true;
      };
      auto load_v = [&](const FwdUnit& u, int j) -> bool {
        const uint32_t s = vc % C::VSTAGES;
        if (vc >= (uint32_t)C::VSTAGES && !warp_wait(bar(C::B_VEMPTY + s), ((vc / C::VSTAGES) - 1) & 1, wd))
          return false;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::TILE);
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(sV + s * C::TILE + c * (kBN * 128), &tm_v, bar(C::B_VFULL + s), c * C::CHUNK_ELEMS, u.h,
                        u.tok0 + j * kBN, pol_kv);
        }
        __syncwarp();
        ++vc;
        return true;
      };
      int unit = blockIdx.x;
      while (ok) {
        FwdUnit U;
        bool have = decode_unit(p, unit, U) && (!FP8 || descale_blocks_ok(p, U, lane));
        while (!have) {  // a unit past the end of its sequence: take the next one
          unit = steal();
          if (unit < 0) break;
          have = decode_unit(p, unit, U) && (!FP8 || descale_blocks_ok(p, U, lane));
        }
        if (!have) break;
        ok = publish(unit) && load_q(U, 0) && load_k(U, 0) && (U.nkv[1] == 0 || load_q(U, 1)) && load_v(U, 0);
        for (int j = 1; ok && j < U.n_iter; ++j) ok = load_k(U, j) && load_v(U, j);
        if (!ok) break;
        unit = steal();
        if (unit < 0) break;
      }
      if (ok) publish(-1);  // no unit left
      // Let every load and scheduler response this warp asked for land before the CTA can exit.
      if (elect_one()) {
        if (c_issued > c_done) drain_wait(bar(C::B_CLC), c_done & 1, p.timeout_ns);
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (qn[t] > 0) drain_wait(bar(C::B_QFULL + t), (qn[t] - 1) & 1, p.timeout_ns);
        for (uint32_t i = kc > (uint32_t)C::KSTAGES ? kc - C::KSTAGES : 0u; i < kc; ++i)
          drain_wait(bar(C::B_KFULL + i % C::KSTAGES), (i / C::KSTAGES) & 1, p.timeout_ns);
        for (uint32_t i = vc > (uint32_t)C::VSTAGES ? vc - C::VSTAGES : 0u; i < vc; ++i)
          drain_wait(bar(C::B_VFULL + i % C::VSTAGES), (i / C::VSTAGES) & 1, p.timeout_ns);
      }
      __syncwarp();
    } else if (warp == 9) {
      // ================================================================ MMA issuer
      // Descriptors are computed once; per instruction only a constant start-address offset
      // (in 16-byte units, no carry out of the 14-bit field: shared addresses stay below 228 KB).
      const uint64_t dq_base = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk_base = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv_base = sdesc_sw128(sV, kBN * 128, 1024);
      uint32_t kc = 0, vc = 0;    // ring positions of the current unit's first K / V tile
      uint32_t qn[2] = {0u, 0u};  // Q tile t loads consumed
      uint32_t pn[2] = {0u, 0u};  // P tiles of Q tile t consumed (all units)
      uint32_t un = 0;            // units read
      bool ok = true;
      auto read_unit = [&](int& unit) -> bool {
        const int s = un & 1;
        if (!warp_wait(bar(C::B_UFULL + s), (un >> 1) & 1, wd)) return false;
        unit = unit_ring[s];
        __syncwarp();
        if (elect_one()) mbar_arrive(bar(C::B_UEMPTY + s));
        __syncwarp();
        ++un;
        return true;
      };
      auto k_wait = [&](uint32_t kpos) -> bool {
        return warp_wait(bar(C::B_KFULL + kpos % C::KSTAGES), (kpos / C::KSTAGES) & 1, wd);
      };
      // S(t, 0) of unit u with its K tile at ring position kpos
      auto first_s = [&](const FwdUnit& u, int t, uint32_t kpos) -> bool {
        if (!warp_wait(bar(C::B_QFULL + t), qn[t] & 1, wd)) return false;
        ++qn[t];
        tc_fence_after();
        if (elect_one()) {
          issue_qk<D, EB, IDESC_S>(tmem + 128u * t, dq_base + ((t * C::TILE) >> 4),
                               dk_base + (((kpos % C::KSTAGES) * C::TILE) >> 4));
          tc_commit(bar(C::B_SFULL + t));
          if (u.nkv[t] == 1) tc_commit(bar(C::B_QEMPTY + t));  // Q tile t is read by no later MMA of u
        }
        __syncwarp();
        return true;
      };
      int cur = -1;
      FwdUnit U;
      ok = read_unit(cur);
      if (ok && cur >= 0) {
        decode_unit(p, cur, U);
        ok = k_wait(0) && first_s(U, 0, 0) && (U.nkv[1] == 0 || first_s(U, 1, 0));
        if (ok && elect_one()) tc_commit(bar(C::B_KEMPTY + 0));  // K_0: both S(·, 0) issued
        __syncwarp();
      }
      while (ok && cur >= 0) {
        // The next unit's S(t, 0) go to the tensor core as soon as Q tile t has issued its last
        // P·V of this unit (MMAs of one thread run in issue order, so S(t, 0) cannot overwrite
        // P(t, last) before that P·V has read it).  Until the unit's last step only non-blocking
        // probes are used: the producer may still be waiting for this warp to free a ring stage.
        int nxt = -1;
        bool nxt_read = false, nx_s0 = false, nx_s1 = false;
        FwdUnit N;
        const uint32_t kn = kc + U.n_iter;  // ring position of the next unit's K_0
        auto prefetch_next = [&](bool done1, bool force) -> bool {
          if (!nxt_read) {
            if (!force && !warp_test(bar(C::B_UFULL + (un & 1)), (un >> 1) & 1)) return true;
            if (!read_unit(nxt)) return false;
            nxt_read = true;
            if (nxt >= 0) decode_unit(p, nxt, N);
          }
          if (nxt < 0) return true;
          if (!nx_s0) {
            if (!force && !(warp_test(bar(C::B_QFULL + 0), qn[0] & 1) &&
                            warp_test(bar(C::B_KFULL + kn % C::KSTAGES), (kn / C::KSTAGES) & 1)))
              return true;
            if (!k_wait(kn) || !first_s(N, 0, kn)) return false;
            nx_s0 = true;
          }
          if (!nx_s1 && (N.nkv[1] == 0 || done1)) {
            if (N.nkv[1] > 0) {
              if (!force && !warp_test(bar(C::B_QFULL + 1), qn[1] & 1)) return true;
              if (!first_s(N, 1, kn)) return false;
            }
            nx_s1 = true;
            if (elect_one()) tc_commit(bar(C::B_KEMPTY + kn % C::KSTAGES));  // both S(·, 0) of the next unit issued
            __syncwarp();
          }
          return true;
        };
        for (int j = 0; ok && j < U.n_iter; ++j) {
          const uint32_t vpos = vc + j;
          const uint64_t dv_s = dv_base + (((vpos % C::VSTAGES) * C::TILE) >> 4);
          const uint32_t kpos1 = kc + j + 1;  // K_{j+1}
          const uint64_t dk_s1 = dk_base + (((kpos1 % C::KSTAGES) * C::TILE) >> 4);
          bool v_ready = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (j >= U.nkv[t]) continue;
            const uint32_t s_tmem = tmem + 128u * t;
            const uint32_t o_tmem = tmem + 256u + (uint32_t)D * t;
            if (!warp_wait(bar(C::B_PFULL + t), pn[t] & 1, wd)) { ok = false; break; }
            ++pn[t];
            if (!v_ready) {
              if (!warp_wait(bar(C::B_VFULL + vpos % C::VSTAGES), (vpos / C::VSTAGES) & 1, wd)) { ok = false; break; }
              v_ready = true;
            }
            tc_fence_after();
            if (elect_one()) {
              issue_pv<EB, IDESC_O>(o_tmem, s_tmem, dv_s, j > 0 ? 1u : 0u);
              if (U.nkv[t] == 1) issue_pv<EB, IDESC_O>(o_tmem, s_tmem + 64u, dv_s, 1u);  // lo part of a split P
              tc_commit(bar(C::B_PVDONE + t));
            }
            __syncwarp();
            if (j + 1 < U.nkv[t]) {
              if (!k_wait(kpos1)) { ok = false; break; }
              tc_fence_after();
              if (elect_one()) {
                issue_qk<D, EB, IDESC_S>(s_tmem, dq_base + ((t * C::TILE) >> 4), dk_s1);
                tc_commit(bar(C::B_SFULL + t));
                if (j + 2 == U.nkv[t]) tc_commit(bar(C::B_QEMPTY + t));  // last S of Q tile t in this unit
              }
              __syncwarp();
            }
          }
          if (!ok) break;
          if (elect_one()) {
            tc_commit(bar(C::B_VEMPTY + vpos % C::VSTAGES));                // V_j: both P·V(·, j) issued
            if (j + 1 < U.n_iter) tc_commit(bar(C::B_KEMPTY + kpos1 % C::KSTAGES));  // K_{j+1}: both S(·, j+1)
          }
          __syncwarp();
          if (j + 1 >= U.nkv[0] && j + 1 < U.n_iter && !prefetch_next(j + 1 >= U.nkv[1], false)) ok = false;
        }
        if (!ok || !prefetch_next(true, true)) break;
        kc += U.n_iter;
        vc += U.n_iter;
        cur = nxt;
        U = N;
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
    regs_inc<200>();
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t tS = tmem + lane_off + 128u * t;
    const uint32_t tO = tmem + lane_off + 256u + (uint32_t)(D * t);
    float c = p.scale_log2;  // per unit when the e4m3 descales are per (sequence, head)
    float2 c2 = make_float2(c, c);
    float o_scale_u = 1.f;   // the unit's v descale in that case (the FP8 instantiation only)
    float kd_next = 1.f, vd_next = 1.f;  // per-block descales of the next KV tile, loaded a tile ahead
    const uint32_t keep_bias = keep_flag_bias(p.drop.t);  // used by the dropout variant only
    uint32_t un = 0;  // units read
    uint32_t sn = 0;  // S tiles of Q tile t consumed (all units)
    bool ok = true;
    while (ok) {
      const int us = un & 1;
      if (!warp_wait(bar(C::B_UFULL + us), (un >> 1) & 1, wd)) break;
      const int unit = unit_ring[us];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_UEMPTY + us));
      ++un;
      if (unit < 0) break;
      FwdUnit U;
      decode_unit(p, unit, U);
      const int my_nkv = U.nkv[t];
      if (my_nkv == 0) continue;
      const int row = U.q0 + t * kBM + 32 * quarter + lane;  // position in the sequence
      const uint32_t drop_bh = (uint32_t)(U.b * p.H + U.h);
      int blk0 = 0;  // first descale block of this sequence (per-block descales)
      if constexpr (FP8) {
        o_scale_u = p.o_scale;
        if (p.descale_blocks > 0) {
          // the producer published the unit only if its blocks lie inside the arrays
          blk0 = descale_block0(p, U, lane);
          // q's descale is that of the 128-row block this Q tile is; k's and v's change per KV tile
          c = p.scale_log2 * __ldg(p.q_descale + (size_t)(blk0 + (U.q0 + t * kBM) / kBM) * p.H + U.h);
          o_scale_u = 1.f;
          kd_next = __ldg(p.k_descale + (size_t)blk0 * p.H + U.h);
          vd_next = __ldg(p.v_descale + (size_t)blk0 * p.H + U.h);
        } else if (p.q_descale != nullptr) {
          const int bh = U.b * p.H + U.h;
          c = p.scale_log2 * (__ldg(p.q_descale + bh) * __ldg(p.k_descale + bh));
          c2 = make_float2(c, c);
          o_scale_u = __ldg(p.v_descale + bh);
        }
      }
      const int key_limit = p.causal ? min(U.L, row + 1) : U.L;
      // A tile whose rows see a single KV tile (the first 128 rows of a causal
      // sequence, or a sequence of at most 128 tokens) averages few values, so
      // the rounding of P to 16 bits would show in O: there P is carried as
      // hi + lo parts and multiplied by V twice.
      const bool split_p = (my_nkv == 1);
      float m_ref = -INFINITY;  // running (possibly stale) max, scaled domain
      float ell = 0.f;
      for (int j = 0; j < my_nkv; ++j) {
        const uint32_t step = sn + j;
        // dropout: the random bytes of this row's 128 keys, word g = keys 4g .. 4g+3 (byte = key offset).
        // One Philox call covers 4 keys × the 4 rows of a lane quad (row mod 4 = lane mod 4): each lane
        // of the quad makes 8 of the tile's 32 calls and the quad exchanges words, so no call is made
        // twice.  Made while S(t, j) is still on the tensor core (measured faster than making each call
        // just before its keys are packed).
        uint32_t rw[DROP ? kBN / 4 : 1];
        if constexpr (DROP) {
          const uint32_t g0 = (uint32_t)(j * kBN) / 4u + (uint32_t)(lane & 3);
#pragma unroll
          for (int m = 0; m < kBN / 16; ++m) {
            const uint4 r4 = philox4x32_10(g0 + 4u * m, (uint32_t)row >> 2, drop_bh, p.drop.offset,
                                           p.drop.seed_lo, p.drop.seed_hi);
            uint32_t x[4] = {r4.x, r4.y, r4.z, r4.w};
            quad_transpose(x, lane);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) rw[4 * m + c4] = x[c4];
          }
        }
        // per-block e4m3 descales of KV tile j: k's folds into this tile's c, v's into P: the tile's P is
        // formed as 2^(c·s − m + log2 v_descale), ℓ takes it divided by v_descale, and m tracks the
        // maximum of c·s + log2 v_descale, so that P stays ≤ 256 and O = Σ P V / ℓ needs no factor
        float lv = 0.f, inv_vd = 1.f;
        if constexpr (FP8) {
          if (p.descale_blocks > 0) {
            const float kd = kd_next, vd = vd_next;
            if (j + 1 < my_nkv) {  // the next tile's, so that the loads are in flight during this tile
              const size_t bi = (size_t)(blk0 + j + 1) * p.H + U.h;
              kd_next = __ldg(p.k_descale + bi);
              vd_next = __ldg(p.v_descale + bi);
            }
            c2 = make_float2(c * kd, c * kd);
            lv = __log2f(vd);
            inv_vd = ex2(-lv);  // 1 / v_descale as P sees it (2^lv), one MUFU operation
          }
        }
        if (!warp_wait(bar(C::B_SFULL + t), step & 1, wd)) { ok = false; break; }
        tc_fence_after();
        // one 128-column load and one 64-column store per tile: fewer, larger tensor-memory accesses
        // slow the MMAs running at the same time less than 32-column pieces of the same bytes
        uint32_t sr[kBN];
        tmem_ld128(tS, sr);
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
        const float m_tile =
            max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * c2.x + lv;
        // raise the reference max only when the tile max exceeds it by more than the threshold
        const float m_new = (m_tile > m_ref + kRescaleThreshold) ? m_tile : m_ref;
        const float alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
        const bool rescale_o = (j > 0) && (m_new != m_ref);
        ell *= alpha;
        m_ref = m_new;
        // a row that has seen no visible key yet keeps m = -inf; its P is 0 either way
        const float neg_m = ((m_ref == -INFINITY) ? 0.f : -m_ref) + lv;
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // pair i = keys 2i, 2i + 1 packed to 16 bits each: dropped keys zeroed (the 1/(1 − p) factor is
        // applied to O at the end; ℓ takes the undropped values)
        auto pair_mask = [&](int i) -> uint32_t {
          if constexpr (!DROP) return ~0u;
          uint32_t m01, m23;
          keep_pair_masks(rw[i >> 1], keep_bias, m01, m23);
          return (i & 1) ? m23 : m01;
        };
        auto drop_pair = [&](uint32_t v, int i) -> uint32_t { return DROP ? v & pair_mask(i) : v; };
        if constexpr (FP8) {
          if (!split_p) {
            // P = 2^(c·s − m), rounded to e4m3, four keys per 32-bit column, written over S.  The MMAs
            // take half as long as at 16 bits, so the exponentials bound the tile: a quarter of them go
            // to the FMA-pipe polynomial (measured 4.8 % faster than all on the MUFU; 1/8 and 3/8 gain
            // less).
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float2 e[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int pi = 2 * i + h;  // pair index
                const float2 x = __ffma2_rn(make_float2(sv[2 * pi], sv[2 * pi + 1]), c2, nm2);
                e[h] = ((kFp8PolyMask >> (pi & 7)) & 1u) ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
                acc[pi & 3] = __fadd2_rn(acc[pi & 3], e[h]);
              }
              pk[i] = pack4_e4m3(e[0].x, e[0].y, e[1].x, e[1].y);
            }
            tmem_st32(tS, pk);
          } else {
            // P = hi + lo, both e4m3: hi in columns [0, 32), lo in [64, 96)
            uint32_t hi[32], lo[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float2 x0 = __ffma2_rn(make_float2(sv[4 * i], sv[4 * i + 1]), c2, nm2);
              const float2 x1 = __ffma2_rn(make_float2(sv[4 * i + 2], sv[4 * i + 3]), c2, nm2);
              const float2 e0 = make_float2(ex2(x0.x), ex2(x0.y));
              const float2 e1 = make_float2(ex2(x1.x), ex2(x1.y));
              acc[(2 * i) & 3] = __fadd2_rn(acc[(2 * i) & 3], e0);
              acc[(2 * i + 1) & 3] = __fadd2_rn(acc[(2 * i + 1) & 3], e1);
              hi[i] = pack4_e4m3(e0.x, e0.y, e1.x, e1.y);
              const float2 h0 = unpack2_e4m3((uint16_t)(hi[i] & 0xFFFFu));
              const float2 h1 = unpack2_e4m3((uint16_t)(hi[i] >> 16));
              lo[i] = pack4_e4m3(e0.x - h0.x, e0.y - h0.y, e1.x - h1.x, e1.y - h1.y);
            }
            tmem_st32(tS, hi);
            tmem_st32(tS + 64u, lo);
          }
        } else if (!split_p && !need_mask && PolyMask<D>::value != 0u) {
          // unmasked tile: part of the exponentials on the FMA pipe, interleaved with the MUFU ones
          uint32_t pk[64];
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float2 x = __ffma2_rn(make_float2(sv[2 * i], sv[2 * i + 1]), c2, nm2);
            float2 e;
            if ((PolyMask<D>::value >> (i & 7)) & 1u) e = exp2_poly2(x);
            else e = make_float2(ex2(x.x), ex2(x.y));
            acc[i & 3] = __fadd2_rn(acc[i & 3], e);
            pk[i] = drop_pair(pack2<BF16>(e.x, e.y), i);
          }
          tmem_st64(tS, pk);
        } else if (!split_p) {
          // P = 2^(c·s − m) on the MUFU (ex2(−inf) = 0 exactly), packed to 16 bits, written over S
          uint32_t pk[64];
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float2 x = __ffma2_rn(make_float2(sv[2 * i], sv[2 * i + 1]), c2, nm2);
            const float2 e = make_float2(ex2(x.x), ex2(x.y));
            acc[i & 3] = __fadd2_rn(acc[i & 3], e);
            pk[i] = drop_pair(pack2<BF16>(e.x, e.y), i);
          }
          tmem_st64(tS, pk);
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
              const uint32_t h2 = pack2<BF16>(e.x, e.y);
              const float2 hf = unpack2<BF16>(h2);
              const uint32_t mk = pair_mask(16 * q + i);
              hi[i] = h2 & mk;
              lo[i] = pack2<BF16>(e.x - hf.x, e.y - hf.y) & mk;
            }
            tmem_st16(tS + 16u * q, hi);
            tmem_st16(tS + 64u + 16u * q, lo);
          }
        }
        const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        if constexpr (FP8) ell += (a.x + a.y) * inv_vd;
        else ell += a.x + a.y;
        if (__any_sync(0xffffffffu, rescale_o)) {
          // The reference max rose (rare past the first tile): O(t) must hold P·V(t, j-1) before it
          // is rescaled, and the rescale must land before P·V(t, j) is issued.
          if (!warp_wait(bar(C::B_PVDONE + t), (step - 1) & 1, wd)) { ok = false; break; }
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
      if (ok && warp_wait(bar(C::B_PVDONE + t), (sn + my_nkv - 1) & 1, wd)) {
        tc_fence_after();
        const bool valid = row < U.L;
        // o_scale: 1/(1 − p) with dropout, v's descale for e4m3
        const float inv = (ell > 0.f) ? (FP8 ? o_scale_u : p.o_scale) / ell : 0.f;
        const size_t obase = ((size_t)(U.tok0 + (valid ? row : 0)) * p.H + U.h) * D;
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
          p.lse[(size_t)(U.tok0 + row) * p.H + U.h] = lse;
        }
      } else {
        ok = false;
      }
      sn += my_nkv;
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

template <int D, bool BF16, bool DROP, bool FP8 = false>
static cudaError_t launch_fwd_t(const Problem& pb, const FwdArgs& a, cudaStream_t stream) {
  using C = FwdCfg<D, FP8 ? 1 : 2>;
  static std::atomic<unsigned long long> configured{0};  // per instantiation, one bit per device
  auto kern = fa_fwd_kernel<D, BF16, DROP, FP8>;
  if (cudaError_t e = set_smem_once(configured, reinterpret_cast<const void*>(kern), C::SMEM_BYTES); e != cudaSuccess)
    return e;
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
  p.scale_log2 = pb.scale * (pb.fp8 ? pb.qk_descale : 1.f) * 1.4426950408889634f;
  p.o_scale = pb.drop.t != 0u ? pb.drop.keep_scale : (pb.fp8 ? pb.v_descale : 1.f);
  p.q_descale = pb.q_descale_bh;
  p.k_descale = pb.k_descale_bh;
  p.v_descale = pb.v_descale_bh;
  p.descale_blocks = pb.descale_blocks;
  p.timeout_ns = pb.timeout_ns;
  p.drop = pb.drop;
  const long long units = (long long)pb.B * pb.H * p.num_qblocks;
  kern<<<dim3((unsigned)units), dim3(kFwdThreads), C::SMEM_BYTES, stream>>>(a.tm_q, a.tm_k, a.tm_v, p);
  return cudaPeekAtLastError();
}

template <bool DROP>
static cudaError_t launch_fwd_d(const Problem& pb, const FwdArgs& a, cudaStream_t stream) {
  if (pb.d == 128)
    return pb.bf16 ? launch_fwd_t<128, true, DROP>(pb, a, stream) : launch_fwd_t<128, false, DROP>(pb, a, stream);
  return pb.bf16 ? launch_fwd_t<64, true, DROP>(pb, a, stream) : launch_fwd_t<64, false, DROP>(pb, a, stream);
}

cudaError_t launch_fwd(const Problem& pb, const FwdArgs& a, cudaStream_t stream) {
  if (pb.fp8) return launch_fwd_t<128, true, false, true>(pb, a, stream);  // e4m3 inputs: d = 128 only
  return pb.drop.t != 0u ? launch_fwd_d<true>(pb, a, stream) : launch_fwd_d<false>(pb, a, stream);
}

}  // namespace fa
