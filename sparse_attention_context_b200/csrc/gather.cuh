// gather.cuh -- 128 gathered query rows into one shared-memory UMMA operand
// tile (K-major, 128B swizzle), by 128 threads.
#pragma once

#include <cstdint>

#include "tc_ptx.cuh"

namespace isa {

// Rows row0 .. row0 + 127 of the row list of head bh (row_idx[bh][n_rows],
// or the identity when row_idx is null) are copied from q [BH, N, D] into
// the tile at shared address `tile`; thread r (0..127) moves the 16-byte
// chunks it * 128 + r, i.e. chunk (it*128 + r) % (D/8) of list row
// (it*128 + r) / (D/8), so each warp reads whole 256-byte row segments.
// List rows past n_rows give zero rows.  An index outside [0, N) gives a
// zero row and ISA_ERR_INVALID_ARG in *status, except -1 when pad_ok (a
// padding entry, skipped silently).  All row indices are loaded first, then
// all rows, then an error is reported: a status write between an index load
// and the row load it feeds would keep the loads of the other rows from
// being in flight together (2 * D/8 memory round trips instead of two).
template <int D>
__device__ __forceinline__ void gather_rows_sw128(const uint16_t* __restrict__ q, const int32_t* __restrict__ row_idx,
                                                  int bh, int n_rows, int N, int row0, int r, uint32_t tile,
                                                  bool pad_ok, int* status) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  int src[CPR];
#pragma unroll
  for (int it = 0; it < CPR; ++it) {
    const int gg = row0 + (it * 128 + r) / CPR;
    src[it] = -1;
    if (gg < n_rows) src[it] = row_idx ? __ldg(row_idx + static_cast<size_t>(bh) * n_rows + gg) : gg;
  }
  uint4 vals[CPR];
#pragma unroll
  for (int it = 0; it < CPR; ++it) {
    const int ch = (it * 128 + r) % CPR;
    vals[it] = make_uint4(0u, 0u, 0u, 0u);
    if (static_cast<unsigned>(src[it]) < static_cast<unsigned>(N))
      vals[it] = __ldg(reinterpret_cast<const uint4*>(q + (static_cast<size_t>(bh) * N + src[it]) * D + ch * 8));
  }
  bool bad = false;
#pragma unroll
  for (int it = 0; it < CPR; ++it) {
    const int gg = row0 + (it * 128 + r) / CPR;
    bad |= gg < n_rows && static_cast<unsigned>(src[it]) >= static_cast<unsigned>(N) && !(pad_ok && src[it] == -1);
  }
  if (bad && status != nullptr) atomicCAS(status, 0, 1 /* ISA_ERR_INVALID_ARG: index out of range, row zeroed */);
#pragma unroll
  for (int it = 0; it < CPR; ++it) {
    const int c = it * 128 + r;
    const int row = c / CPR, ch = c % CPR;
    st_shared_v4(tile + (ch >> 3) * (128 * 128) + sw128(row, ch & 7), vals[it].x, vals[it].y, vals[it].z,
                 vals[it].w);
  }
}

}  // namespace isa
