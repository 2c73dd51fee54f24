// isa_abi.cu -- the C ABI declared in include/isa.h: argument validation,
// workspace layout, tensor-map encoding and the launch sequence of every
// ISA stage.  Host code only; the arithmetic lives in the kernel files.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "isa.h"
#include "isa_internal.h"

namespace isa {
namespace {

struct Dims {
  int B, H, BH, N_src, N_ctx, N, d, blk, nSB, nCB, nB, nBp, n_keep, n_route, n_rb, nK, nKpad, nChunks;
  float scale;
};

struct WsLayout {
  size_t Kbar, Vbar, ksel, qksplit, partial, sal, Khi, Klo, Vb, bias2, sharp, kept, routed, taylor, rblk,
      rrows, opart, mlpart, total;
  int split_ctas;  // key-split partial CTAs the workspace holds
};

// SMs of the current device (the key-split partial buffers hold one CTA per
// SM); 148 when no device is visible (sizing on a host without a GPU).
int split_ctas_for_device() {
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) !=
                                               cudaSuccess || nsm <= 0) {
    cudaGetLastError();
    return 148;
  }
  return nsm;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// ceil(frac*n - g) in [0, n], guard g = min(1e-6*n, 0.5): absorbs the float32
// rounding of frac (0.2f*40560 = 8112.0001 counts 8112) and never takes a
// whole unit off an exact product.
int guarded_count(float frac, int n) {
  const double g = std::min(1e-6 * n, 0.5);
  const double v = std::ceil(static_cast<double>(frac) * n - g);
  return static_cast<int>(std::min<double>(std::max<double>(v, 0.0), n));
}
int keep_count(float keep, int nCB) { return guarded_count(keep, nCB); }
int route_count(float rho, int N) { return guarded_count(rho, N); }

int check_shape(const isa_shape* s, Dims* o) {
  if (s == nullptr) return ISA_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->N_src < 1 || s->N_ctx < 0) return ISA_ERR_INVALID_ARG;
  if (!(s->keep >= 0.f && s->keep <= 1.f) || !(s->rho >= 0.f && s->rho <= 1.f)) return ISA_ERR_INVALID_ARG;
  if (!std::isfinite(s->scale)) return ISA_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return ISA_ERR_UNSUPPORTED;
  if (s->block != 64 && s->block != 128) return ISA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(s->B) * s->H;
  const long long N = static_cast<long long>(s->N_src) + s->N_ctx;
  if (BH > 65535) return ISA_ERR_UNSUPPORTED;
  if (BH * (N + 4096) >= INT_MAX) return ISA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  Dims d{};
  d.B = s->B;
  d.H = s->H;
  d.BH = static_cast<int>(BH);
  d.N_src = s->N_src;
  d.N_ctx = s->N_ctx;
  d.N = static_cast<int>(N);
  d.d = s->d;
  d.blk = s->block;
  d.nSB = (d.N_src + d.blk - 1) / d.blk;
  d.nCB = (d.N_ctx + d.blk - 1) / d.blk;
  if (d.nCB > kTopkCap) return ISA_ERR_UNSUPPORTED;
  d.nB = d.nSB + d.nCB;
  d.n_keep = keep_count(s->keep, d.nCB);
  d.n_route = route_count(s->rho, d.N);
  d.n_rb = route_count(s->rho, d.nB);  // block-granular grouping: same rule over the nB query blocks
  d.nK = d.nSB + d.n_keep;
  d.nKpad = (d.nK + 127) / 128 * 128;
  d.nBp = (d.nB + 127) / 128 * 128;
  d.nChunks = d.nBp / 128;  // saliency row tiles
  d.scale = s->scale > 0.f ? s->scale : 1.0f / std::sqrt(static_cast<float>(d.d));
  *o = d;
  return ISA_OK;
}

WsLayout layout(const Dims& d) {
  WsLayout L{};
  size_t off = kCtlBytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const size_t BH = d.BH;
  L.Kbar = take(BH * d.nB * d.d * 4);
  L.Vbar = take(BH * d.nB * d.d * 4);
  L.ksel = take(BH * std::max(d.n_keep, 1) * 4);
  L.qksplit = take(4 * BH * d.nBp * d.d * 2);
  L.partial = take(BH * d.nChunks * std::max(d.nCB, 1) * 4);
  L.sal = take(BH * std::max(d.nCB, 1) * 4);
  L.Khi = take(BH * d.nKpad * d.d * 2);
  L.Klo = take(BH * d.nKpad * d.d * 2);
  L.Vb = take(BH * d.nKpad * d.d * 2);
  L.bias2 = take(BH * d.nKpad * 4);
  L.sharp = take(BH * d.N * 4);
  L.kept = take(BH * std::max(d.n_keep, 1) * 4);
  L.routed = take(BH * std::max(d.n_route, 1) * 4);
  L.taylor = take(BH * std::max(d.N - d.n_route, 1) * 4);
  L.rblk = take(BH * std::max(d.n_rb, 1) * 4);
  L.rrows = take(BH * std::max(d.n_rb * d.blk, 1) * 4);
  L.split_ctas = split_ctas_for_device();
  L.opart = take(static_cast<size_t>(L.split_ctas) * 256 * d.d * 4);
  L.mlpart = take(static_cast<size_t>(L.split_ctas) * 256 * 8);
  L.total = off;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || !aligned16(ws)) return ISA_ERR_INVALID_ARG;
  if (ws_bytes < need) return ISA_ERR_WORKSPACE;
  return ISA_OK;
}

int cuda_status(cudaError_t e) { return record_cuda_status(e); }

// --- tensor maps (driver entry point fetched once through the runtime)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Common pieces of the stage launches.
struct Ctx {
  Dims d;
  WsLayout L;
  void* ws;
  cudaStream_t st;
  int* status() const { return at<int>(ws, kStatusOffset); }
  const int* inject() const { return at<int>(ws, kInjectOffset); }
};

FlashParams base_params(const Ctx& c) {
  FlashParams p{};
  p.o_part = at<float>(c.ws, c.L.opart);
  p.ml_part = at<float2>(c.ws, c.L.mlpart);
  p.split_capacity = c.L.split_ctas;
  p.N = c.d.N;
  p.N_src = c.d.N_src;
  p.N_ctx = c.d.N_ctx;
  p.blk = c.d.blk;
  p.nSB = c.d.nSB;
  p.n_keep = c.d.n_keep;
  p.scale_log2 = c.d.scale * 1.4426950408889634f;
  p.status = c.status();
  p.inject = c.inject();
  return p;
}

int run_preselect(const Ctx& c, const uint16_t* q, const uint16_t* k, const uint16_t* v, int32_t* kept,
                  float* sal_user) {
  const Dims& d = c.d;
  uint16_t* split = at<uint16_t>(c.ws, c.L.qksplit);
  const size_t plane = static_cast<size_t>(d.BH) * d.nBp * d.d;  // Qhi, Qlo, Khi, Klo
  cudaError_t e = launch_pool(q, k, v, nullptr, at<float>(c.ws, c.L.Kbar),
                              at<float>(c.ws, c.L.Vbar), split, d.BH, d.N_src, d.N_ctx, d.d, d.blk, c.st);
  if (e == cudaSuccess)
    e = launch_saliency_tc(split, split + plane, split + 2 * plane, split + 3 * plane,
                           at<float>(c.ws, c.L.partial), d.BH, d.N_src, d.N_ctx, d.d, d.blk, d.scale, c.status(),
                           c.st);
  if (e == cudaSuccess)
    e = launch_select_ctx(at<float>(c.ws, c.L.partial), d.nChunks, at<float>(c.ws, c.L.sal), sal_user, kept, d.BH,
                          d.N_src, d.N_ctx, d.blk, d.n_keep, c.st);
  if (e == cudaSuccess)
    e = launch_pool_kept_v(v, kept, at<int32_t>(c.ws, c.L.ksel), at<float>(c.ws, c.L.Vbar), d.BH, d.N_src, d.N_ctx,
                           d.d, d.blk, d.n_keep, c.st);
  return cuda_status(e);
}

int run_build_kept(const Ctx& c, const int32_t* kept) {
  const Dims& d = c.d;
  return cuda_status(launch_build_kept(at<float>(c.ws, c.L.Kbar), at<float>(c.ws, c.L.Vbar), kept,
                                       at<int32_t>(c.ws, c.L.ksel), at<uint16_t>(c.ws, c.L.Khi), at<uint16_t>(c.ws, c.L.Klo),
                                       at<uint16_t>(c.ws, c.L.Vb), at<float>(c.ws, c.L.bias2), d.BH, d.N_src,
                                       d.N_ctx, d.d, d.blk, d.n_keep, d.nKpad, c.status(), c.st));
}

int run_route(const Ctx& c, const uint16_t* q, const int32_t* kept, int32_t* routed, int32_t* taylor,
              float* sharp_user) {
  const Dims& d = c.d;
  int rc = run_build_kept(c, kept);
  if (rc != ISA_OK) return rc;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return ISA_ERR_CUDA;
  CUtensorMap tmHi, tmLo;
  if (!make_tmap_bf16(&tmHi, at<uint16_t>(c.ws, c.L.Khi), static_cast<uint64_t>(d.BH) * d.nKpad, d.d, 128) ||
      !make_tmap_bf16(&tmLo, at<uint16_t>(c.ws, c.L.Klo), static_cast<uint64_t>(d.BH) * d.nKpad, d.d, 128))
    return ISA_ERR_CUDA;
  float* sharp = sharp_user ? sharp_user : at<float>(c.ws, c.L.sharp);
  FlashParams p = base_params(c);
  p.q = q;
  p.sharp = sharp;
  p.row_idx = nullptr;
  p.n_rows = d.N;
  p.n_kv_tiles = d.nKpad / 128;
  p.kv_rows_per_head = d.nKpad;
  p.bias2 = at<float>(c.ws, c.L.bias2);
  cudaError_t e = launch_flash(d.d, 128, MODE_SHARP, tmHi, tmLo, p, d.BH, c.st);
  if (e == cudaSuccess) e = launch_route(sharp, routed, taylor, d.BH, d.N, d.n_route, c.status(), c.st);
  return cuda_status(e);
}

// Stages 2 and 4 in one pass over q: sharpness and the Taylor output of
// every row (fused kernel), then routing.
int run_route_taylor(const Ctx& c, const uint16_t* q, const int32_t* kept, int32_t* routed, int32_t* taylor,
                     float* sharp_user, uint16_t* out, bool route = true) {
  const Dims& d = c.d;
  int rc = run_build_kept(c, kept);
  if (rc != ISA_OK) return rc;
  CUtensorMap tmQ, tmHi, tmLo, tmVb, tmO;
  const uint64_t kv_rows = static_cast<uint64_t>(d.BH) * d.nKpad;
  if (!make_tmap_bf16(&tmQ, q, static_cast<uint64_t>(d.BH) * d.N, d.d, 128) ||
      !make_tmap_bf16_3d(&tmO, out, d.BH, d.N, d.d, 128) ||
      !make_tmap_bf16(&tmHi, at<uint16_t>(c.ws, c.L.Khi), kv_rows, d.d, 128) ||
      !make_tmap_bf16(&tmLo, at<uint16_t>(c.ws, c.L.Klo), kv_rows, d.d, 128) ||
      !make_tmap_bf16(&tmVb, at<uint16_t>(c.ws, c.L.Vb), kv_rows, d.d, 128))
    return ISA_ERR_CUDA;
  float* sharp = sharp_user ? sharp_user : at<float>(c.ws, c.L.sharp);
  FlashParams p = base_params(c);
  p.q = q;
  p.out = out;
  p.sharp = sharp;
  p.row_idx = nullptr;
  p.n_rows = d.N;
  p.n_kv_tiles = d.nKpad / 128;
  p.kv_rows_per_head = d.nKpad;
  p.bias2 = at<float>(c.ws, c.L.bias2);
  cudaError_t e = launch_fused(d.d, tmQ, tmHi, tmLo, tmVb, tmO, p, d.BH, c.st);
  if (e == cudaSuccess && route) e = launch_route(sharp, routed, taylor, d.BH, d.N, d.n_route, c.status(), c.st);
  return cuda_status(e);
}

// Full attention for an explicit row list of n_rows entries per (b, h)
// (entries of -1 are padding: computed on zeros, never stored).
int run_full_rows(const Ctx& c, const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* kept,
                  const int32_t* rows, int n_rows, uint16_t* out) {
  const Dims& d = c.d;
  cudaError_t e = cudaSuccess;
  if (n_rows > 0) {
    CUtensorMap tmK, tmV;
    if (!make_tmap_bf16(&tmK, k, static_cast<uint64_t>(d.BH) * d.N, d.d, d.blk) ||
        !make_tmap_bf16(&tmV, v, static_cast<uint64_t>(d.BH) * d.N, d.d, d.blk))
      return ISA_ERR_CUDA;
    FlashParams p = base_params(c);
    p.q = q;
    p.out = out;
    p.row_idx = rows;
    p.n_rows = n_rows;
    p.kept_ctx = kept;
    p.n_kv_tiles = d.nSB + d.n_keep;
    p.kv_rows_per_head = d.N;
    e = launch_attn2(d.d, d.blk, MODE_FULL, tmK /* Q is gathered by threads */, tmK, tmV, p, d.BH, c.st);
  }
  return cuda_status(e);
}

int run_full(const Ctx& c, const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* kept,
             const int32_t* routed, uint16_t* out) {
  return run_full_rows(c, q, k, v, kept, routed, c.d.n_route, out);
}

// Block-granular variant of run_route_taylor: the same fused sharpness +
// Taylor pass over every row, then whole query blocks are routed.
int run_route_blocks_taylor(const Ctx& c, const uint16_t* q, const int32_t* kept, int32_t* routed_blk,
                            int32_t* routed_rows, float* score_user, float* sharp_user, uint16_t* out) {
  const Dims& d = c.d;
  float* sharp = sharp_user ? sharp_user : at<float>(c.ws, c.L.sharp);
  int rc = run_route_taylor(c, q, kept, nullptr, nullptr, sharp, out, /*route=*/false);
  if (rc != ISA_OK) return rc;
  return cuda_status(launch_route_blocks(sharp, routed_blk, routed_rows, score_user, d.BH, d.N_src, d.N_ctx, d.blk,
                                         d.n_rb, c.status(), c.st));
}

int run_taylor(const Ctx& c, const uint16_t* q, const int32_t* kept, const int32_t* taylor, uint16_t* out,
               bool rebuild_kept) {
  const Dims& d = c.d;
  if (d.N - d.n_route <= 0) return ISA_OK;
  if (rebuild_kept) {
    const int rc = run_build_kept(c, kept);
    if (rc != ISA_OK) return rc;
  }
  cudaError_t e = cudaSuccess;
  {
    CUtensorMap tmK, tmV;
    if (!make_tmap_bf16(&tmK, at<uint16_t>(c.ws, c.L.Khi), static_cast<uint64_t>(d.BH) * d.nKpad, d.d, 128) ||
        !make_tmap_bf16(&tmV, at<uint16_t>(c.ws, c.L.Vb), static_cast<uint64_t>(d.BH) * d.nKpad, d.d, 128))
      return ISA_ERR_CUDA;
    FlashParams p = base_params(c);
    p.q = q;
    p.out = out;
    p.row_idx = taylor;
    p.n_rows = d.N - d.n_route;
    p.n_kv_tiles = d.nKpad / 128;
    p.kv_rows_per_head = d.nKpad;
    p.bias2 = at<float>(c.ws, c.L.bias2);
    e = launch_flash(d.d, 128, MODE_TAYLOR, tmK, tmV, p, d.BH, c.st);
  }
  return cuda_status(e);
}

// First-order Taylor for the taylor_idx rows: the correction matrices of
// the kept blocks into cws, then the first-order pass.  The gathered kept
// operands (Khi, Vb, bias2) must be current (run_build_kept).
int run_taylor1(const Ctx& c, const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* kept,
                const int32_t* taylor, uint16_t* out, uint16_t* cws) {
  const Dims& d = c.d;
  CUtensorMap tmK, tmV;
  if (!make_tmap_bf16(&tmK, k, static_cast<uint64_t>(d.BH) * d.N, d.d, d.blk) ||
      !make_tmap_bf16(&tmV, v, static_cast<uint64_t>(d.BH) * d.N, d.d, d.blk))
    return ISA_ERR_CUDA;
  cudaError_t e = launch_cbuild(d.d, tmK, tmV, at<float>(c.ws, c.L.Kbar), at<float>(c.ws, c.L.Vbar), kept, cws, d.BH,
                                d.N_src, d.N_ctx, d.blk, d.n_keep, c.status(), c.st);
  if (e != cudaSuccess || d.N - d.n_route <= 0) return cuda_status(e);
  CUtensorMap tmKb, tmVb, tmC;
  const uint64_t kv_rows = static_cast<uint64_t>(d.BH) * d.nKpad;
  if (!make_tmap_bf16(&tmKb, at<uint16_t>(c.ws, c.L.Khi), kv_rows, d.d, 128) ||
      !make_tmap_bf16(&tmVb, at<uint16_t>(c.ws, c.L.Vb), kv_rows, d.d, 128) ||
      !make_tmap_bf16(&tmC, cws, static_cast<uint64_t>(d.BH) * d.nK * d.d, d.d, d.d))
    return ISA_ERR_CUDA;
  FlashParams p = base_params(c);
  p.q = q;
  p.out = out;
  p.row_idx = taylor;
  p.n_rows = d.N - d.n_route;
  p.n_kv_tiles = d.nKpad / 128;
  p.kv_rows_per_head = d.nKpad;
  p.bias2 = at<float>(c.ws, c.L.bias2);
  return cuda_status(launch_taylor1(d.d, tmKb, tmVb, tmC, p, d.nK, d.scale, d.BH, c.st));
}

size_t taylor1_bytes(const Dims& d) {
  return align256(static_cast<size_t>(d.BH) * d.nK * d.d * d.d * 2);
}

int run_attn(const Ctx& c, const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* kept,
             const int32_t* routed, const int32_t* taylor, uint16_t* out, bool rebuild_kept) {
  int rc = run_full(c, q, k, v, kept, routed, out);
  if (rc == ISA_OK) rc = run_taylor(c, q, kept, taylor, out, rebuild_kept);
  return rc;
}

int make_ctx(const isa_shape* shape, void* ws, size_t ws_bytes, void* stream, Ctx* c) {
  int rc = check_shape(shape, &c->d);
  if (rc != ISA_OK) return rc;
  c->L = layout(c->d);
  rc = check_ws(ws, ws_bytes, c->L.total);
  if (rc != ISA_OK) return rc;
  c->ws = ws;
  c->st = static_cast<cudaStream_t>(stream);
  return ISA_OK;
}

bool tensors_ok(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p == nullptr || !aligned16(p)) return false;
  return true;
}

}  // namespace

thread_local cudaError_t g_last_cuda_error = cudaSuccess;  // reported by isa_last_error()

bool nvtx_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("ISA_NVTX");
    return e != nullptr && e[0] != '\0' && std::strcmp(e, "0") != 0;
  }();
  return on;
}

int record_cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ISA_OK;
  g_last_cuda_error = e;
  return ISA_ERR_CUDA;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, int D, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, int BH, int N, int D, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace isa

using namespace isa;

extern "C" {

int isa_n_keep(const isa_shape* shape) {
  Dims d;
  return check_shape(shape, &d) == ISA_OK ? d.n_keep : -1;
}

int isa_n_route(const isa_shape* shape) {
  Dims d;
  return check_shape(shape, &d) == ISA_OK ? d.n_route : -1;
}

int isa_n_route_blocks(const isa_shape* shape) {
  Dims d;
  return check_shape(shape, &d) == ISA_OK ? d.n_rb : -1;
}

size_t isa_workspace_size(const isa_shape* shape) {
  Dims d;
  if (check_shape(shape, &d) != ISA_OK) return 0;
  return layout(d).total;
}

int isa_preselect_ctx(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      int32_t* kept_ctx_idx, float* saliency, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_preselect_ctx");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, k, v})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (saliency != nullptr && !aligned16(saliency)) return ISA_ERR_INVALID_ARG;
  return run_preselect(c, q, k, v, kept_ctx_idx, saliency);
}

int isa_route_queries(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx, int32_t* routed_idx,
                      int32_t* taylor_idx, float* sharpness, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_route_queries");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.n_route > 0 && (routed_idx == nullptr || !aligned16(routed_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.N - c.d.n_route > 0 && (taylor_idx == nullptr || !aligned16(taylor_idx))) return ISA_ERR_INVALID_ARG;
  if (sharpness != nullptr && !aligned16(sharpness)) return ISA_ERR_INVALID_ARG;
  return run_route(c, q, kept_ctx_idx, routed_idx, taylor_idx, sharpness);
}

int isa_attn_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 const int32_t* kept_ctx_idx, const int32_t* routed_idx, const int32_t* taylor_idx, uint16_t* out,
                 void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_attn_fwd");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.n_route > 0 && (routed_idx == nullptr || !aligned16(routed_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.N - c.d.n_route > 0 && (taylor_idx == nullptr || !aligned16(taylor_idx))) return ISA_ERR_INVALID_ARG;
  return run_attn(c, q, k, v, kept_ctx_idx, routed_idx, taylor_idx, out, true);
}

int isa_route_taylor_fwd(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx,
                         int32_t* routed_idx, int32_t* taylor_idx, float* sharpness, uint16_t* out, void* ws,
                         size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_route_taylor_fwd");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, out})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.n_route > 0 && (routed_idx == nullptr || !aligned16(routed_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.N - c.d.n_route > 0 && (taylor_idx == nullptr || !aligned16(taylor_idx))) return ISA_ERR_INVALID_ARG;
  if (sharpness != nullptr && !aligned16(sharpness)) return ISA_ERR_INVALID_ARG;
  return run_route_taylor(c, q, kept_ctx_idx, routed_idx, taylor_idx, sharpness, out);
}

int isa_full_attn_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const int32_t* kept_ctx_idx, const int32_t* routed_idx, uint16_t* out, void* ws,
                      size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_full_attn_fwd");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.n_route > 0 && (routed_idx == nullptr || !aligned16(routed_idx))) return ISA_ERR_INVALID_ARG;
  return run_full(c, q, k, v, kept_ctx_idx, routed_idx, out);
}

int isa_taylor_attn_fwd(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx,
                        const int32_t* taylor_idx, uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_taylor_attn_fwd");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, out})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.N - c.d.n_route > 0 && (taylor_idx == nullptr || !aligned16(taylor_idx))) return ISA_ERR_INVALID_ARG;
  return run_taylor(c, q, kept_ctx_idx, taylor_idx, out, true);
}

int isa_forward(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_forward");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  int32_t* kept = at<int32_t>(ws, c.L.kept);
  int32_t* routed = at<int32_t>(ws, c.L.routed);
  int32_t* taylor = at<int32_t>(ws, c.L.taylor);
  {
    NvtxRange r("isa_forward: pre-selection");
    rc = run_preselect(c, q, k, v, kept, nullptr);
  }
  if (rc == ISA_OK) {
    NvtxRange r("isa_forward: sharpness + Taylor + route");
    rc = run_route_taylor(c, q, kept, routed, taylor, nullptr, out);
  }
  if (rc == ISA_OK) {
    NvtxRange r("isa_forward: full attention");
    rc = run_full(c, q, k, v, kept, routed, out);
  }
  return rc;
}

int isa_route_blocks_taylor_fwd(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx,
                                int32_t* routed_blk_idx, int32_t* routed_rows, float* block_score, float* sharpness,
                                uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_route_blocks_taylor_fwd");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (c.d.nB > kRouteBlocksCap) return ISA_ERR_UNSUPPORTED;
  if (!tensors_ok({q, out})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.n_rb > 0 && !tensors_ok({routed_blk_idx, routed_rows})) return ISA_ERR_INVALID_ARG;
  if ((block_score != nullptr && !aligned16(block_score)) || (sharpness != nullptr && !aligned16(sharpness)))
    return ISA_ERR_INVALID_ARG;
  return run_route_blocks_taylor(c, q, kept_ctx_idx, routed_blk_idx, routed_rows, block_score, sharpness, out);
}

int isa_full_attn_rows_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const int32_t* kept_ctx_idx, const int32_t* row_idx, int n_rows, uint16_t* out,
                           void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_full_attn_rows_fwd");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (n_rows < 0) return ISA_ERR_INVALID_ARG;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (n_rows > 0 && (row_idx == nullptr || !aligned16(row_idx))) return ISA_ERR_INVALID_ARG;
  if (static_cast<long long>(c.d.BH) * n_rows >= INT_MAX) return ISA_ERR_UNSUPPORTED;
  return run_full_rows(c, q, k, v, kept_ctx_idx, row_idx, n_rows, out);
}

int isa_forward_blocks(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_forward_blocks");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (c.d.nB > kRouteBlocksCap) return ISA_ERR_UNSUPPORTED;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  int32_t* kept = at<int32_t>(ws, c.L.kept);
  int32_t* rblk = at<int32_t>(ws, c.L.rblk);
  int32_t* rrows = at<int32_t>(ws, c.L.rrows);
  rc = run_preselect(c, q, k, v, kept, nullptr);
  if (rc == ISA_OK) rc = run_route_blocks_taylor(c, q, kept, rblk, rrows, nullptr, nullptr, out);
  if (rc == ISA_OK) rc = run_full_rows(c, q, k, v, kept, rrows, c.d.n_rb * c.d.blk, out);
  return rc;
}

size_t isa_taylor1_workspace_size(const isa_shape* shape) {
  Dims d;
  if (check_shape(shape, &d) != ISA_OK) return 0;
  return taylor1_bytes(d);
}

int isa_taylor1_attn_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* kept_ctx_idx, const int32_t* taylor_idx, uint16_t* out, void* ws,
                         size_t ws_bytes, void* cws, size_t cws_bytes, void* stream) {
  NvtxRange nvtx_("isa_taylor1_attn_fwd");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  if (c.d.n_keep > 0 && (kept_ctx_idx == nullptr || !aligned16(kept_ctx_idx))) return ISA_ERR_INVALID_ARG;
  if (c.d.N - c.d.n_route > 0 && (taylor_idx == nullptr || !aligned16(taylor_idx))) return ISA_ERR_INVALID_ARG;
  rc = check_ws(cws, cws_bytes, taylor1_bytes(c.d));
  if (rc != ISA_OK) return rc;
  if (static_cast<long long>(c.d.BH) * c.d.nK * c.d.d >= INT_MAX) return ISA_ERR_UNSUPPORTED;
  rc = run_build_kept(c, kept_ctx_idx);
  if (rc != ISA_OK) return rc;
  return run_taylor1(c, q, k, v, kept_ctx_idx, taylor_idx, out, static_cast<uint16_t*>(cws));
}

int isa_forward_taylor1(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        uint16_t* out, void* ws, size_t ws_bytes, void* cws, size_t cws_bytes, void* stream) {
  NvtxRange nvtx_("isa_forward_taylor1");
  Ctx c;
  int rc = make_ctx(shape, ws, ws_bytes, stream, &c);
  if (rc != ISA_OK) return rc;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  rc = check_ws(cws, cws_bytes, taylor1_bytes(c.d));
  if (rc != ISA_OK) return rc;
  if (static_cast<long long>(c.d.BH) * c.d.nK * c.d.d >= INT_MAX) return ISA_ERR_UNSUPPORTED;
  int32_t* kept = at<int32_t>(ws, c.L.kept);
  int32_t* routed = at<int32_t>(ws, c.L.routed);
  int32_t* taylor = at<int32_t>(ws, c.L.taylor);
  rc = run_preselect(c, q, k, v, kept, nullptr);
  // the fused sharpness pass (it also gathers the kept operands) writes
  // 0-th order rows that the first-order pass then overwrites: cheaper than
  // the stage-by-stage sharpness kernel
  if (rc == ISA_OK) rc = run_route_taylor(c, q, kept, routed, taylor, nullptr, out);
  if (rc == ISA_OK) rc = run_full(c, q, k, v, kept, routed, out);
  if (rc == ISA_OK) rc = run_taylor1(c, q, k, v, kept, taylor, out, static_cast<uint16_t*>(cws));
  return rc;
}

size_t isa_dense_workspace_size(int d) {
  if (d != 64 && d != 128) return 0;
  const int nsm = split_ctas_for_device();
  return kCtlBytes + 4096 + align256(static_cast<size_t>(nsm) * 256 * d * 4) + align256(static_cast<size_t>(nsm) * 256 * 8);
}

int isa_dense_attn_fwd(int B, int H, int N, int d, float scale, const uint16_t* q, const uint16_t* k,
                       const uint16_t* v, uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("isa_dense_attn_fwd");
  if (B < 1 || H < 1 || N < 1 || !std::isfinite(scale)) return ISA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ISA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 65535 || BH * (static_cast<long long>(N) + 128) >= INT_MAX) return ISA_ERR_UNSUPPORTED;
  if (!tensors_ok({q, k, v, out})) return ISA_ERR_INVALID_ARG;
  int rc = check_ws(ws, ws_bytes, kCtlBytes);
  if (rc != ISA_OK) return rc;
  // key-split partials after the control block, as many CTAs as fit
  const size_t per = split_bytes_per_cta(d);
  const int cap = ws_bytes > kCtlBytes + 4096 ? static_cast<int>((ws_bytes - kCtlBytes - 4096) / per) : 0;
  CUtensorMap tmQ, tmK, tmV;
  if (!make_tmap_bf16(&tmQ, q, static_cast<uint64_t>(BH) * N, d, 128) ||
      !make_tmap_bf16(&tmK, k, static_cast<uint64_t>(BH) * N, d, 128) ||
      !make_tmap_bf16(&tmV, v, static_cast<uint64_t>(BH) * N, d, 128))
    return ISA_ERR_CUDA;
  FlashParams p{};
  p.q = q;
  p.out = out;
  p.row_idx = nullptr;
  p.n_rows = N;
  p.N = N;
  p.n_kv_tiles = (N + 127) / 128;
  p.kv_rows_per_head = N;
  p.scale_log2 = (scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d))) * 1.4426950408889634f;
  p.status = at<int>(ws, kStatusOffset);
  p.inject = at<int>(ws, kInjectOffset);
  if (cap > 0) {
    p.o_part = at<float>(ws, kCtlBytes);
    p.ml_part = at<float2>(ws, align256(kCtlBytes + static_cast<size_t>(cap) * 256 * d * 4));
    p.split_capacity = cap;
  }
  return cuda_status(launch_attn2(d, 128, MODE_DENSE, tmQ, tmK, tmV, p, static_cast<int>(BH),
                                  static_cast<cudaStream_t>(stream)));
}

int isa_read_device_status(void* ws, void* stream) {
  if (ws == nullptr) return ISA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ISA_ERR_CUDA;
  if (cudaMemcpyAsync(&h, at<int>(ws, kStatusOffset), sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return ISA_ERR_CUDA;
  if (cudaMemsetAsync(at<int>(ws, kStatusOffset), 0, sizeof(int), st) != cudaSuccess) return ISA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ISA_ERR_CUDA;
  return h;
}

const char* isa_last_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no CUDA error recorded" : cudaGetErrorString(g_last_cuda_error);
}

const char* isa_status_string(int status) {
  switch (status) {
    case ISA_OK: return "ok";
    case ISA_ERR_INVALID_ARG: return "invalid argument";
    case ISA_ERR_UNSUPPORTED: return "unsupported shape";
    case ISA_ERR_WORKSPACE: return "workspace too small";
    case ISA_ERR_CUDA: return "CUDA error";
    case ISA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
