// isa_internal.h -- launch interfaces shared by the kernel files and the
// host ABI (isa_abi.cu).  Not part of the public C ABI.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

namespace isa {

constexpr int kStatusOffset = 0;   // int32 in the workspace control block
constexpr int kInjectOffset = 4;   // int32 fault-injection word (tests)
constexpr int kCtlBytes = 256;
constexpr int kTopkCap = 4096;     // max context blocks per head the selection kernel holds
constexpr int kRouteBlocksCap = 16384;  // max query blocks per head of the block grouping
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s

enum FlashMode { MODE_DENSE = 0, MODE_FULL = 1, MODE_TAYLOR = 2, MODE_SHARP = 3 };

// Arguments of the tcgen05 attention engine (one CTA = 128 query rows of
// one (b, h); grid = (ceil(n_rows/128), B*H)).
struct FlashParams {
  const uint16_t* q;      // [BH, N, D] bf16
  uint16_t* out;          // [BH, N, D] bf16 (DENSE / FULL / TAYLOR)
  float* sharp;           // [BH, N] fp32 (SHARP)
  const int* row_idx;     // [BH, n_rows] gathered query rows, or null (contiguous)
  int n_rows;             // query rows per head handled by this launch
  int N;                  // tokens per head
  int N_src, N_ctx, blk;  // FULL: segment sizes and block size (== BN)
  int nSB;                // FULL: number of source blocks
  const int* kept_ctx;    // FULL: [BH, n_keep] kept context blocks
  int n_keep;
  int n_kv_tiles;         // key tiles per head
  int kv_rows_per_head;   // rows of the K/V tensor maps per head
  const float* bias2;     // TAYLOR / SHARP: [BH, kv_rows_per_head] log2 cnt (-inf pad)
  float scale_log2;       // s * log2(e)
  int* status;            // device status word or null
  const int* inject;      // device fault-injection word or null
  // two-tile engine only: work items are (b*H + h) * pairs_per_head + pair
  // (256 query rows each); a launch covers items from item_base.
  int item_base;
  int pairs_per_head;
  // key-split launch (split_pieces > 0): CTA g handles item
  // item_base + g / split_pieces over key tiles [piece*nT/pieces,
  // (piece+1)*nT/pieces) and writes unnormalised partials instead of out.
  int split_pieces;
  float* o_part;          // [CTAs, 256, D] fp32 partial accumulators
  float2* ml_part;        // [CTAs, 256] (reference max in log2 units, sum)
  int split_capacity;     // CTAs the partial buffers hold (0 = no split)
};

// ISA_OK for cudaSuccess; otherwise records e as the calling thread's last
// CUDA error (isa_last_error) and returns ISA_ERR_CUDA.
int record_cuda_status(cudaError_t e);

// NVTX ranges around the C entry points, for timelines in a profiler.  Off
// unless the environment variable ISA_NVTX is set to anything but "0" (read
// once per process); when off, a range costs one branch.
bool nvtx_enabled();
struct NvtxRange {
  bool on;
  explicit NvtxRange(const char* name) : on(nvtx_enabled()) {
    if (on) nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Bytes per CTA of key-split partials for head dim D.
inline size_t split_bytes_per_cta(int D) { return 256ull * (static_cast<size_t>(D) * 4 + 8); }

// Tensor map over [BH, N, D] bf16 (D innermost), box = 64 columns x box_rows
// rows x 1 matrix, 128-byte swizzle: rows past N of a matrix are clipped.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, int BH, int N, int D, int box_rows);
// Tensor map over a [rows, D] bf16 row-major matrix, box = 64 columns x
// box_rows rows, 128-byte swizzle.  Returns false if encoding fails.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, int D, int box_rows);

// One-tile engine (flash.cu): SHARP and TAYLOR modes; grid (ceil(n_rows/128), BH).
cudaError_t launch_flash(int D, int BN, int mode, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const FlashParams& p, int BH, cudaStream_t st);
// Two-tile engine (flash2.cu): DENSE and FULL modes; 256-row work items,
// whole waves in one launch plus a key-split tail and its merge.  tmQ is
// read in DENSE (contiguous rows, box 64 x 128); FULL gathers Q by threads.
// Persistent sharpness + Taylor kernel (fused.cu): one CTA per SM looping
// over 256-row items; tmQ over [BH*N, D] (box 128 rows), tmKhi / tmKlo / tmV
// over the gathered kept operands [BH*kv_rows_per_head, D] (box 128 rows),
// tmO the 3-D map of out (make_tmap_bf16_3d, box 128 rows).
cudaError_t launch_fused(int D, const CUtensorMap& tmQ, const CUtensorMap& tmKhi, const CUtensorMap& tmKlo,
                         const CUtensorMap& tmV, const CUtensorMap& tmO, const FlashParams& p, int BH,
                         cudaStream_t st);
cudaError_t launch_attn2(int D, int BN, int mode, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                         const CUtensorMap& tmV, const FlashParams& p, int BH, cudaStream_t st);

// Stage-1 kernels.  launch_pool writes fp32 Kbar, Vbar of the source blocks
// (Qbar too unless it is null) and bf16 hi / lo of Qbar and Kbar
// into QKsplit: four [BH, nBp, D] arrays (Qhi, Qlo, Khi, Klo), nBp = nB
// rounded up to 128, pad rows left unwritten.  launch_saliency_tc: partial
// [BH, nBp/128, nCB] column sums per 128-row tile; launch_select_ctx adds
// the n_chunks partial rows in order.
cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, float* Qbar, float* Kbar,
                        float* Vbar, uint16_t* QKsplit, int BH, int N_src, int N_ctx, int D, int blk,
                        cudaStream_t st);
// Vbar rows of the kept context blocks (pool_kernel leaves the context rows
// of Vbar unwritten), once kept [BH, n_keep] is known; the set is recorded
// in ksel [BH, n_keep], which launch_build_kept checks its kept set against.
cudaError_t launch_pool_kept_v(const uint16_t* v, const int32_t* kept, int32_t* ksel, float* Vbar, int BH,
                               int N_src, int N_ctx, int D, int blk, int n_keep, cudaStream_t st);
cudaError_t launch_saliency_tc(const uint16_t* Qhi, const uint16_t* Qlo, const uint16_t* Khi, const uint16_t* Klo,
                               float* partial, int BH, int N_src, int N_ctx, int D, int blk, float scale,
                               int* status, cudaStream_t st);
cudaError_t launch_select_ctx(const float* partial, int n_chunks, float* sal_ws, float* sal_user, int32_t* kept,
                              int BH, int N_src, int N_ctx, int blk, int n_keep, cudaStream_t st);
cudaError_t launch_build_kept(const float* Kbar, const float* Vbar, const int32_t* kept, const int32_t* ksel,
                              uint16_t* Khi, uint16_t* Klo, uint16_t* Vb, float* bias2, int BH, int N_src, int N_ctx,
                              int D, int blk, int n_keep, int nKpad, int* status, cudaStream_t st);
cudaError_t launch_route(const float* sharp, int32_t* routed, int32_t* taylor, int BH, int N, int n_route,
                         int* status, cudaStream_t st);
// First-order Taylor variant (taylor1.cu).  cbuild: C_b = sum_j (k_j - Kbar_b)
// v_j^T of every kept block, bf16 [BH, nK, D, D] row-major; tmK / tmV over
// k / v [BH*N, D] with box rows = blk.  taylor1: the rows of p.row_idx;
// tmK / tmV over the gathered kept Kbar (bf16 hi) / Vbar [BH*nKpad, D] (box
// 128 rows), tmC over Cout [BH*nK*D, D] (box D rows); p.bias2 = log2 cnt.
cudaError_t launch_cbuild(int D, const CUtensorMap& tmK, const CUtensorMap& tmV, const float* Kbar,
                          const float* Vbar, const int32_t* kept, uint16_t* Cout, int BH, int N_src, int N_ctx,
                          int blk, int n_keep, int* status, cudaStream_t st);
cudaError_t launch_taylor1(int D, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmC,
                           const FlashParams& p, int nK, float scale, int BH, cudaStream_t st);
// Block-granular grouping (route_blocks.cu): routed_blk [BH, n_rb] ascending
// block indices, routed_rows [BH, n_rb*blk] rows of those blocks (-1 pads),
// score_out [BH, nB] block mean sharpness or null.
cudaError_t launch_route_blocks(const float* sharp, int32_t* routed_blk, int32_t* routed_rows, float* score_out,
                                int BH, int N_src, int N_ctx, int blk, int n_rb, int* status, cudaStream_t st);

}  // namespace isa
