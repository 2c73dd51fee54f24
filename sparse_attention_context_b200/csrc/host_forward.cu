// host_forward.cu -- isa_forward_host: the whole ISA forward on host
// buffers, with the PCIe copies pipelined against the kernels (see
// include/isa.h).
//
// Every (b, h) of the forward is an independent unit (selection, routing
// and both attention paths are decided per head), so the B*H heads are
// taken in `groups` consecutive slices.  Slice g goes through three
// streams: its q, k, v are copied in on stream_in, the forward runs on
// stream_compute (isa_forward on the slice's sub-shape, B = 1, H = heads of
// the slice), its output is copied out on stream_out.  The caller's staging
// buffer holds a ring of R = min(groups, 3) slots of q, k, v, out for one
// slice each, so the copy-in of slice g, the forward of slice g-1 and the
// copy-out of slice g-2 can run at once.  Events order the ring:
//   copy-in g   waits until the forward of slice g-R has read its slot;
//   forward g   waits for copy-in g and for the copy-out of slice g-R
//               (which reads the slot's out buffer the forward overwrites);
//   copy-out g  waits for forward g.
// One event per (slot, role) suffices: each is waited on before it is
// recorded again, in host order.  Nothing is allocated on the device; the
// events are created and destroyed per call.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "isa.h"
#include "isa_internal.h"

namespace {

constexpr int kRing = 3;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct HostPlan {
  int BH, G, R, smax;        // heads, slices, ring slots, heads of the largest slice
  size_t slice_elems;        // elements of one tensor of the largest slice
  size_t ws_bytes;           // isa_forward workspace of the largest slice
  size_t off_slots;          // first slot, after the workspace
  size_t slot_bytes;         // q, k, v, out of one slice
  size_t total;
};

int plan(const isa_shape* s, int groups, HostPlan* p) {
  if (s == nullptr) return ISA_ERR_INVALID_ARG;
  // an invalid or unsupported shape: isa_forward's shape check says which
  if (isa_workspace_size(s) == 0) return isa_forward(s, nullptr, nullptr, nullptr, nullptr, nullptr, 0, nullptr);
  const int BH = s->B * s->H;
  int G = groups;
  if (G <= 0) G = BH >= 8 ? BH / 2 : 1;  // default: two heads a slice
  G = std::min(G, BH);
  const int smax = (BH + G - 1) / G;      // slices of floor/ceil(BH/G) heads
  isa_shape sub = *s;
  sub.B = 1;
  sub.H = smax;
  const size_t N = static_cast<size_t>(s->N_src) + s->N_ctx;
  p->BH = BH;
  p->G = G;
  p->R = std::min(G, kRing);
  p->smax = smax;
  p->slice_elems = static_cast<size_t>(smax) * N * s->d;
  p->ws_bytes = align256(isa_workspace_size(&sub));
  p->off_slots = p->ws_bytes;
  p->slot_bytes = 4 * align256(p->slice_elems * 2);
  p->total = p->off_slots + static_cast<size_t>(p->R) * p->slot_bytes;
  return p->ws_bytes > 0 ? ISA_OK : ISA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" size_t isa_host_staging_size(const isa_shape* shape, int groups) {
  HostPlan p;
  return plan(shape, groups, &p) == ISA_OK ? p.total : 0;
}

extern "C" int isa_forward_host(const isa_shape* shape, const uint16_t* hq, const uint16_t* hk, const uint16_t* hv,
                                uint16_t* hout, void* staging, size_t staging_bytes, int groups,
                                void* stream_compute, void* stream_in, void* stream_out) {
  isa::NvtxRange nvtx_("isa_forward_host");
  HostPlan P;
  int rc = plan(shape, groups, &P);
  if (rc != ISA_OK) return rc;
  if (hq == nullptr || hk == nullptr || hv == nullptr || hout == nullptr || staging == nullptr)
    return ISA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(staging) & 15u) != 0) return ISA_ERR_INVALID_ARG;
  if (staging_bytes < P.total) return ISA_ERR_WORKSPACE;

  cudaStream_t sc = static_cast<cudaStream_t>(stream_compute);
  cudaStream_t si = stream_in != nullptr ? static_cast<cudaStream_t>(stream_in) : sc;
  cudaStream_t so = stream_out != nullptr ? static_cast<cudaStream_t>(stream_out) : sc;
  char* base = static_cast<char*>(staging);
  void* ws = base;  // the slices' workspace (control block first), reused slice after slice
  const size_t N = static_cast<size_t>(shape->N_src) + shape->N_ctx;
  const size_t head_elems = N * shape->d;
  const size_t tbytes = align256(P.slice_elems * 2);

  cudaEvent_t ev_start, ev_fin, ev_in[kRing], ev_comp[kRing], ev_out[kRing];
  int made = 0;
  cudaEvent_t* all[2 + 3 * kRing] = {&ev_start, &ev_fin};
  for (int r = 0; r < kRing; ++r) {
    all[2 + 3 * r] = &ev_in[r];
    all[3 + 3 * r] = &ev_comp[r];
    all[4 + 3 * r] = &ev_out[r];
  }
  cudaError_t e = cudaSuccess;
  for (; made < 2 + 3 * kRing && e == cudaSuccess; ++made) {
    e = cudaEventCreateWithFlags(all[made], cudaEventDisableTiming);
    if (e != cudaSuccess) break;
  }
  auto destroy = [&] {
    for (int i = 0; i < made; ++i) cudaEventDestroy(*all[i]);
  };
  if (e != cudaSuccess) {
    destroy();
    return isa::record_cuda_status(e);
  }
  auto fail = [&](cudaError_t err) {
    destroy();
    return isa::record_cuda_status(err);
  };

  // the copy streams start after whatever the compute stream holds (a
  // previous call's use of the staging buffer included)
  if ((e = cudaMemsetAsync(ws, 0, 256, sc)) != cudaSuccess) return fail(e);
  if ((e = cudaEventRecord(ev_start, sc)) != cudaSuccess) return fail(e);
  if (si != sc && (e = cudaStreamWaitEvent(si, ev_start, 0)) != cudaSuccess) return fail(e);
  if (so != sc && (e = cudaStreamWaitEvent(so, ev_start, 0)) != cudaSuccess) return fail(e);

  const uint16_t* hsrc[3] = {hq, hk, hv};
  for (int g = 0; g < P.G; ++g) {
    const int h0 = static_cast<int>(static_cast<long long>(P.BH) * g / P.G);
    const int h1 = static_cast<int>(static_cast<long long>(P.BH) * (g + 1) / P.G);
    const int slot = g % P.R;
    char* sb = base + P.off_slots + static_cast<size_t>(slot) * P.slot_bytes;
    uint16_t* d[4];
    for (int t = 0; t < 4; ++t) d[t] = reinterpret_cast<uint16_t*>(sb + t * tbytes);
    const size_t off = static_cast<size_t>(h0) * head_elems;
    const size_t bytes = static_cast<size_t>(h1 - h0) * head_elems * 2;
    // copy-in (slot free once the forward of slice g - R has run)
    if (g >= P.R && (e = cudaStreamWaitEvent(si, ev_comp[slot], 0)) != cudaSuccess) return fail(e);
    for (int t = 0; t < 3; ++t)
      if ((e = cudaMemcpyAsync(d[t], hsrc[t] + off, bytes, cudaMemcpyDefault, si)) != cudaSuccess) return fail(e);
    if ((e = cudaEventRecord(ev_in[slot], si)) != cudaSuccess) return fail(e);
    // forward of the slice
    if ((e = cudaStreamWaitEvent(sc, ev_in[slot], 0)) != cudaSuccess) return fail(e);
    if (g >= P.R && (e = cudaStreamWaitEvent(sc, ev_out[slot], 0)) != cudaSuccess) return fail(e);
    isa_shape sub = *shape;
    sub.B = 1;
    sub.H = h1 - h0;
    rc = isa_forward(&sub, d[0], d[1], d[2], d[3], ws, P.ws_bytes, sc);
    if (rc != ISA_OK) {
      destroy();
      return rc;
    }
    if ((e = cudaEventRecord(ev_comp[slot], sc)) != cudaSuccess) return fail(e);
    // copy-out
    if ((e = cudaStreamWaitEvent(so, ev_comp[slot], 0)) != cudaSuccess) return fail(e);
    if ((e = cudaMemcpyAsync(hout + off, d[3], bytes, cudaMemcpyDefault, so)) != cudaSuccess) return fail(e);
    if ((e = cudaEventRecord(ev_out[slot], so)) != cudaSuccess) return fail(e);
  }
  // the compute stream ends after the last copy-out
  if ((e = cudaEventRecord(ev_fin, so)) != cudaSuccess) return fail(e);
  if (so != sc && (e = cudaStreamWaitEvent(sc, ev_fin, 0)) != cudaSuccess) return fail(e);
  destroy();  // released once the recorded work completes
  return ISA_OK;
}
