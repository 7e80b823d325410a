// fa_api.cu — the C ABI of libfa_b200.so: argument validation, TMA tensor-map
// encoding, launch of the sm_100a kernels, and the device status word.
#include <cmath>
#include <cstdio>
#include <cstring>

#include "../../include/fa.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

static uint64_t g_watchdog_ns = 4000000000ull;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool encode_tmap(CUtensorMap* map, const void* base, int T, int H, int d, bool bf16, int rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// e4m3 [T, H, d] as bytes: one 128-byte box per row (d = 128), 128-byte swizzle.
bool encode_tmap_e4m3(CUtensorMap* map, const void* base, int T, int H, int d, int rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)H * d};
  const cuuint32_t box[3] = {128, 1, (cuuint32_t)rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_f32(CUtensorMap* map, const void* base, int T, int H, int d, int rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4};
  const cuuint32_t box[3] = {32, 1, (cuuint32_t)rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Checks the size arguments shared by every entry point and fills `pb`.
static int make_problem(Problem* pb, int B, int H, int N, int d, float scale, int causal, const int32_t* cu,
                        int total_tokens, int dtype, bool need_scale) {
  if (B < 1 || H < 1 || N < 1 || total_tokens < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (need_scale && (!std::isfinite(scale) || !(scale > 0.f))) return FA_ERR_INVALID_ARG;
  if (cu == nullptr) {
    if ((long long)B * N != (long long)total_tokens) return FA_ERR_INVALID_ARG;
  } else if ((reinterpret_cast<uintptr_t>(cu) & 3u) != 0) {
    return FA_ERR_INVALID_ARG;
  }
  // grid and index limits
  const long long qblocks = (N + 255) / 256;
  if ((long long)B * H * qblocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if ((long long)total_tokens * H * d > (1LL << 40)) return FA_ERR_UNSUPPORTED;
  pb->B = B;
  pb->H = H;
  pb->N = N;
  pb->d = d;
  pb->T = total_tokens;
  pb->scale = scale;
  pb->causal = causal;
  pb->cu_seqlens = cu;
  pb->bf16 = (dtype == FA_BF16);
  pb->timeout_ns = g_watchdog_ns;
  pb->drop = Dropout{0u, 1.f, 0u, 0u, 0u};
  pb->fp8 = false;
  pb->qk_descale = 1.f;
  pb->v_descale = 1.f;
  pb->q_descale_bh = pb->k_descale_bh = pb->v_descale_bh = nullptr;
  pb->descale_blocks = 0;
  return FA_OK;
}

// Dropout on P (see fa.h): threshold byte t = round(256·p) clamped to 255, keep scale 256/(256 − t).
static int set_dropout(Problem* pb, float p, uint64_t seed, uint32_t offset) {
  if (!(p >= 0.f && p < 1.f)) return FA_ERR_INVALID_ARG;  // also rejects NaN
  const double t = std::floor((double)p * 256.0 + 0.5);
  pb->drop.t = (uint32_t)(t > 255.0 ? 255.0 : t);
  pb->drop.keep_scale = (float)(256.0 / (256.0 - (double)pb->drop.t));
  pb->drop.seed_lo = (uint32_t)(seed & 0xFFFFFFFFull);
  pb->drop.seed_hi = (uint32_t)(seed >> 32);
  pb->drop.offset = offset;
  return FA_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static size_t workspace_bytes(int T, int H, int d) {
  return align256((size_t)T * H * d * sizeof(float)) + align256((size_t)T * H * sizeof(float));
}

static int set_workspace(BwdArgs* a, void* ws, size_t ws_bytes, int T, int H, int d) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(T, H, d)) return FA_ERR_INVALID_ARG;
  a->dq_acc = reinterpret_cast<float*>(ws);
  a->delta = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + align256((size_t)T * H * d * sizeof(float)));
  return FA_OK;
}

static int map_launch(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

}  // namespace fa

namespace fa {

static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                    float scale, int causal, const int32_t* cu_seqlens, int total_tokens, int dtype, bool dropout,
                    float dropout_p, uint64_t seed, uint32_t offset, fa_stream_t stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, true);
  if (st != FA_OK) return st;
  if (dropout && (st = set_dropout(&pb, dropout_p, seed, offset)) != FA_OK) return st;
  FwdArgs a;
  if (!encode_tmap(&a.tm_q, q, pb.T, H, d, pb.bf16, 128) || !encode_tmap(&a.tm_k, k, pb.T, H, d, pb.bf16, 128) ||
      !encode_tmap(&a.tm_v, v, pb.T, H, d, pb.bf16, 128))
    return FA_ERR_UNSUPPORTED;
  a.o = o;
  a.lse = lse;
  return map_launch(launch_fwd(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

static int bwd_main_impl(const void* q, const void* k, const void* v, const float* lse, const void* dO, void* dk,
                         void* dv, int B, int H, int N, int d, float scale, int causal, const int32_t* cu_seqlens,
                         int total_tokens, int dtype, bool dropout, float dropout_p, uint64_t seed, uint32_t offset,
                         void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(lse) || !aligned16(dO) || !aligned16(dk) ||
      !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, true);
  if (st != FA_OK) return st;
  if (dropout && (st = set_dropout(&pb, dropout_p, seed, offset)) != FA_OK) return st;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if ((st = set_workspace(&a, workspace, workspace_bytes_, pb.T, H, d)) != FA_OK) return st;
  // Q and dO stream in tiles of bq rows (the main kernel's query step); K and V in 128-row tiles
  const int bq = bwd_q_tile_rows(d, dropout);
  if (!encode_tmap(&a.tm_q, q, pb.T, H, d, pb.bf16, bq) || !encode_tmap(&a.tm_k, k, pb.T, H, d, pb.bf16, 128) ||
      !encode_tmap(&a.tm_v, v, pb.T, H, d, pb.bf16, 128) || !encode_tmap(&a.tm_do, dO, pb.T, H, d, pb.bf16, bq) ||
      !encode_tmap_f32(&a.tm_dq, a.dq_acc, pb.T, H, d, bwd_dq_box_rows(d, dropout)))
    return FA_ERR_UNSUPPORTED;
  a.q = q;
  a.k = k;
  a.lse = lse;
  a.dO = dO;
  a.dk = dk;
  a.dv = dv;
  return map_launch(launch_bwd_main(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace fa

using namespace fa;

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, const int32_t* cu_seqlens, int total_tokens, int dtype, fa_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, false, 0.f, 0, 0, stream);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
               float scale, int causal, const int32_t* cu_seqlens, int total_tokens, float q_descale,
               float k_descale, float v_descale, fa_stream_t stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_INVALID_ARG;
  Problem pb;
  // sizes and scale are checked as for a bf16 call (the output is bf16)
  int st = make_problem(&pb, B, H, N, d, scale, causal, cu_seqlens, total_tokens, FA_BF16, true);
  if (st != FA_OK) return st;
  for (float ds : {q_descale, k_descale, v_descale})
    if (!std::isfinite(ds) || !(ds > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  pb.fp8 = true;
  pb.qk_descale = q_descale * k_descale;
  pb.v_descale = v_descale;
  if (!std::isfinite(pb.scale * pb.qk_descale) || !(pb.scale * pb.qk_descale > 0.f)) return FA_ERR_INVALID_ARG;
  FwdArgs a;
  if (!encode_tmap_e4m3(&a.tm_q, q, pb.T, H, d, 128) || !encode_tmap_e4m3(&a.tm_k, k, pb.T, H, d, 128) ||
      !encode_tmap_e4m3(&a.tm_v, v, pb.T, H, d, 128))
    return FA_ERR_UNSUPPORTED;
  a.o = o;
  a.lse = lse;
  return map_launch(launch_fwd(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

int fa_fwd_fp8_per_head(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                        float scale, int causal, const int32_t* cu_seqlens, int total_tokens, const float* q_descale,
                        const float* k_descale, const float* v_descale, fa_stream_t stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_INVALID_ARG;
  if (!aligned4(q_descale) || !aligned4(k_descale) || !aligned4(v_descale)) return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, scale, causal, cu_seqlens, total_tokens, FA_BF16, true);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  pb.fp8 = true;
  pb.q_descale_bh = q_descale;
  pb.k_descale_bh = k_descale;
  pb.v_descale_bh = v_descale;
  FwdArgs a;
  if (!encode_tmap_e4m3(&a.tm_q, q, pb.T, H, d, 128) || !encode_tmap_e4m3(&a.tm_k, k, pb.T, H, d, 128) ||
      !encode_tmap_e4m3(&a.tm_v, v, pb.T, H, d, 128))
    return FA_ERR_UNSUPPORTED;
  a.o = o;
  a.lse = lse;
  return map_launch(launch_fwd(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

int fa_fwd_fp8_per_block(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                         int d, float scale, int causal, const int32_t* cu_seqlens, int total_tokens,
                         const float* q_descale, const float* k_descale, const float* v_descale, int num_blocks,
                         fa_stream_t stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_INVALID_ARG;
  if (!aligned4(q_descale) || !aligned4(k_descale) || !aligned4(v_descale)) return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, scale, causal, cu_seqlens, total_tokens, FA_BF16, true);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  // dense: every sequence has ceil(N / 128) blocks; varlen: checked per sequence on the device
  const long long dense_blocks = (long long)B * ((N + 127) / 128);
  if (num_blocks < 1 || (cu_seqlens == nullptr && num_blocks < dense_blocks)) return FA_ERR_INVALID_ARG;
  pb.fp8 = true;
  pb.q_descale_bh = q_descale;
  pb.k_descale_bh = k_descale;
  pb.v_descale_bh = v_descale;
  pb.descale_blocks = num_blocks;
  FwdArgs a;
  if (!encode_tmap_e4m3(&a.tm_q, q, pb.T, H, d, 128) || !encode_tmap_e4m3(&a.tm_k, k, pb.T, H, d, 128) ||
      !encode_tmap_e4m3(&a.tm_v, v, pb.T, H, d, 128))
    return FA_ERR_UNSUPPORTED;
  a.o = o;
  a.lse = lse;
  return map_launch(launch_fwd(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                   float scale, int causal, const int32_t* cu_seqlens, int total_tokens, int dtype, float dropout_p,
                   uint64_t seed, uint32_t offset, fa_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, true, dropout_p, seed,
                  offset, stream);
}

size_t fa_bwd_workspace_bytes(int total_tokens, int H, int d) {
  if (total_tokens < 1 || H < 1 || (d != 64 && d != 128)) return 0;
  return workspace_bytes(total_tokens, H, d);
}

int fa_bwd_preprocess(const void* o, const void* dO, int B, int H, int N, int d, const int32_t* cu_seqlens,
                      int total_tokens, int dtype, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  if (!aligned16(o) || !aligned16(dO)) return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, 1.f, 0, cu_seqlens, total_tokens, dtype, false);
  if (st != FA_OK) return st;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if ((st = set_workspace(&a, workspace, workspace_bytes_, pb.T, H, d)) != FA_OK) return st;
  a.o = o;
  a.dO = dO;
  return map_launch(launch_bwd_pre(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

int fa_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dO, void* dk, void* dv,
                int B, int H, int N, int d, float scale, int causal, const int32_t* cu_seqlens, int total_tokens,
                int dtype, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return bwd_main_impl(q, k, v, lse, dO, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, false,
                       0.f, 0, 0, workspace, workspace_bytes_, stream);
}

int fa_bwd_postprocess(void* dq, int B, int H, int N, int d, float scale, const int32_t* cu_seqlens,
                       int total_tokens, int dtype, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  if (!aligned16(dq)) return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, scale, 0, cu_seqlens, total_tokens, dtype, true);
  if (st != FA_OK) return st;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if ((st = set_workspace(&a, workspace, workspace_bytes_, pb.T, H, d)) != FA_OK) return st;
  a.dq = dq;
  return map_launch(launch_bwd_post(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
           void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, const int32_t* cu_seqlens,
           int total_tokens, int dtype, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  // validate everything before launching anything
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, true);
  if (st != FA_OK) return st;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if ((st = set_workspace(&a, workspace, workspace_bytes_, pb.T, H, d)) != FA_OK) return st;
  st = fa_bwd_preprocess(o, dO, B, H, N, d, cu_seqlens, total_tokens, dtype, workspace, workspace_bytes_, stream);
  if (st != FA_OK) return st;
  st = fa_bwd_main(q, k, v, lse, dO, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, workspace,
                   workspace_bytes_, stream);
  if (st != FA_OK) return st;
  return fa_bwd_postprocess(dq, B, H, N, d, scale, cu_seqlens, total_tokens, dtype, workspace, workspace_bytes_,
                            stream);
}

int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                   const int32_t* cu_seqlens, int total_tokens, int dtype, float dropout_p, uint64_t seed,
                   uint32_t offset, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  // validate everything before launching anything
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, true);
  if (st != FA_OK) return st;
  if ((st = set_dropout(&pb, dropout_p, seed, offset)) != FA_OK) return st;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if ((st = set_workspace(&a, workspace, workspace_bytes_, pb.T, H, d)) != FA_OK) return st;
  // D = rowsum(dO ∘ O) holds with dropout too (O is the dropped output), so pre and post are shared
  st = fa_bwd_preprocess(o, dO, B, H, N, d, cu_seqlens, total_tokens, dtype, workspace, workspace_bytes_, stream);
  if (st != FA_OK) return st;
  st = bwd_main_impl(q, k, v, lse, dO, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, true,
                     dropout_p, seed, offset, workspace, workspace_bytes_, stream);
  if (st != FA_OK) return st;
  return fa_bwd_postprocess(dq, B, H, N, d, scale, cu_seqlens, total_tokens, dtype, workspace, workspace_bytes_,
                            stream);
}

int fa_attn_merge(float* acc_o, float* acc_lse, const void* part_o, const float* part_lse, void* out, int T, int H,
                  int d, int dtype, int first, fa_stream_t stream) {
  if (!aligned16(acc_o) || !aligned4(acc_lse) || !aligned16(part_o) || !aligned4(part_lse)) return FA_ERR_INVALID_ARG;
  if (out != nullptr && !aligned16(out)) return FA_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || (d != 64 && d != 128) || (first != 0 && first != 1)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if ((long long)T * H * d > (1LL << 40)) return FA_ERR_UNSUPPORTED;
  return map_launch(launch_merge(acc_o, acc_lse, part_o, part_lse, out, (long long)T * H, d, dtype == FA_BF16, first,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

int fa_accumulate(float* acc, const void* part, void* out, long long n, int dtype, int first, fa_stream_t stream) {
  if (!aligned16(acc) || (part != nullptr && !aligned16(part)) || (out != nullptr && !aligned16(out)))
    return FA_ERR_INVALID_ARG;
  if (n < 8 || (n & 7) != 0 || (first != 0 && first != 1)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  return map_launch(launch_accumulate(acc, part, out, n, dtype == FA_BF16, first, reinterpret_cast<cudaStream_t>(stream)));
}

size_t fa_decode_workspace_bytes(int B, int H, int Nk, int d) {
  if (B < 1 || H < 1 || Nk < 1 || (d != 64 && d != 128)) return 0;
  const size_t slots = (size_t)B * H * decode_chunks(Nk);
  return align256(slots * d * sizeof(float)) + align256(slots * 2 * sizeof(float));
}

int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nk, int d,
              float scale, const int32_t* cu_seqlens_k, int total_keys, int dtype, void* workspace,
              size_t workspace_bytes_, fa_stream_t stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_INVALID_ARG;
  Problem pb;
  int st = make_problem(&pb, B, H, Nk, d, scale, 0, cu_seqlens_k, total_keys, dtype, true);
  if (st != FA_OK) return st;
  if (B > 65535 || H > 65535) return FA_ERR_UNSUPPORTED;  // grid y / z
  const size_t need = fa_decode_workspace_bytes(B, H, Nk, d);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes_ < need)
    return FA_ERR_INVALID_ARG;
  DecodeArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  const size_t slots = (size_t)B * H * decode_chunks(Nk);
  a.part_o = reinterpret_cast<float*>(workspace);
  a.part_ml = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + align256(slots * d * sizeof(float)));
  return map_launch(launch_decode(pb, a, reinterpret_cast<cudaStream_t>(stream)));
}

int fa_check_device_status(fa_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  return h;
}

void fa_set_watchdog_ns(uint64_t ns) { g_watchdog_ns = ns < 1000000ull ? 1000000ull : ns; }

int fa_watchdog_selftest(uint64_t timeout_ns, fa_stream_t stream) {
  if (timeout_ns < 1000000ull) timeout_ns = 1000000ull;
  if (timeout_ns > 10000000000ull) return FA_ERR_INVALID_ARG;
  int st = fa_check_device_status(stream);  // start from a clean word
  if (st == FA_ERR_CUDA) return st;
  if (launch_watchdog_selftest(timeout_ns, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  return fa_check_device_status(stream);
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    default: return "FA_UNKNOWN_STATUS";
  }
}

const char* fa_version(void) { return "fa_b200 0.1 (sm_100a)"; }

}  // extern "C"
