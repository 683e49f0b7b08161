// bsa_host.cu -- the whole path from host buffers: frame-major q, k, v and the
// dense block mask in host memory in, attention output and LSE in host memory
// out, with the copies overlapped with the kernels.
//
// Heads are independent problems (each has its own mask, CRM rows, token
// permutation and softmax), so the B*H heads are cut into chunks and run as a
// three-stage pipeline on three streams:
//   copy-in  stream:  chunk c's q, k, v and mask, host -> device
//   compute  stream:  bsa_pack_mask, bsa_tile_permute (q, k, v), bsa_forward,
//                     bsa_tile_unpermute of chunk c  (the caller's stream)
//   copy-out stream:  chunk c's output and LSE, device -> host
// Chunk c uses buffer slot c % 2, so while chunk c computes, chunk c + 1 is
// copied in and chunk c - 1 is copied out (separate copy engines each way).
// Events order the reuse of a slot: the copy-in of chunk c waits for the
// compute of chunk c - 2 (it read the slot's inputs), and the compute of chunk
// c waits for the copy-out of chunk c - 2 (it read the slot's outputs).  The
// two auxiliary streams are created once per device and joined back into the
// caller's stream, so the call is ordered on that stream like any other.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "bsa.h"
#include "bsa_internal.h"

namespace {

constexpr int kSlots = 2;
constexpr int kMaxDevices = 64;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte offsets of one slot's buffers inside the workspace.
struct SlotLayout {
  size_t qf, kf, vf;      // frame-major inputs   [hc, N, d] bf16
  size_t qp, kp, vp, op;  // tile-major           [hc, n_pad, d] bf16
  size_t of;              // frame-major output   [hc, N, d] bf16
  size_t lse;             // [hc, n_pad] fp32
  size_t dense;           // [hc, nb, nb] uint8
  size_t bits, counts, offsets, schedule, pack_ws;
  size_t pack_ws_bytes;
  size_t bytes;           // whole slot
};

SlotLayout slot_layout(int hc, int64_t n, int64_t n_pad, int d, int nb) {
  SlotLayout L{};
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at += align256(bytes);
    return here;
  };
  const size_t frame = size_t(hc) * n * d * 2, tiled = size_t(hc) * n_pad * d * 2;
  const int words = (nb + 31) / 32;
  L.qf = take(frame);
  L.kf = take(frame);
  L.vf = take(frame);
  L.qp = take(tiled);
  L.kp = take(tiled);
  L.vp = take(tiled);
  L.op = take(tiled);
  L.of = take(frame);
  L.lse = take(size_t(hc) * n_pad * 4);
  L.dense = take(size_t(hc) * nb * nb);
  L.bits = take(size_t(hc) * nb * words * 4);
  L.counts = take(size_t(hc) * nb * 4);
  L.offsets = take((size_t(hc) * nb + 1) * 4);
  L.schedule = take(size_t(hc) * nb * 4);
  L.pack_ws_bytes = bsa_pack_mask_workspace(1, hc, nb, nb);
  L.pack_ws = take(L.pack_ws_bytes);
  L.bytes = at;
  return L;
}

// About 16 chunks: at 720p with 40 heads, chunks of 3 heads measured fastest
// (52.1 ms per step; 2 heads 52.6, 5 heads 53.4, 1 head 60.8, 10 heads 60.6):
// small enough that filling and draining the pipeline is short, large enough
// that every chunk's forward fills the GPU.
int default_chunk(int BH) { return (BH + 15) / 16; }

// Auxiliary streams and per-slot events, created once per device.
struct DeviceCtx {
  bool ready = false;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t h2d_done[kSlots] = {}, comp_done[kSlots] = {}, d2h_done[kSlots] = {};
};

std::mutex g_ctx_mutex;
DeviceCtx g_ctx[kMaxDevices];

DeviceCtx* device_ctx() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_ctx_mutex);
  DeviceCtx& c = g_ctx[dev];
  if (!c.ready) {
    const unsigned ev_flags = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&c.copy_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c.copy_out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.start, ev_flags) != cudaSuccess)
      return nullptr;
    for (int s = 0; s < kSlots; ++s)
      if (cudaEventCreateWithFlags(&c.h2d_done[s], ev_flags) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.comp_done[s], ev_flags) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.d2h_done[s], ev_flags) != cudaSuccess)
        return nullptr;
    c.ready = true;
  }
  return &c;
}

}  // namespace

extern "C" size_t bsa_attention_host_workspace(int B, int H, int T, int Hs, int Ws, int d,
                                               int block, int heads_per_chunk) {
  if (B <= 0 || H <= 0 || T <= 0 || Hs <= 0 || Ws <= 0 || d <= 0 || block <= 0) return 0;
  const int BH = B * H;
  const int hc = heads_per_chunk > 0 ? (heads_per_chunk < BH ? heads_per_chunk : BH)
                                     : default_chunk(BH);
  const int64_t n = int64_t(T) * Hs * Ws;
  const int64_t n_pad = (n + block - 1) / block * block;
  return kSlots * slot_layout(hc, n, n_pad, d, int(n_pad / block)).bytes;
}

extern "C" bsa_status bsa_attention_host(const void* q, const void* k, const void* v,
                                         const uint8_t* mask, void* out, float* lse, int B, int H,
                                         int T, int Hs, int Ws, int d, int tt, int th, int tw,
                                         int block, float softmax_scale, int heads_per_chunk,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !mask || !out || !lse || !workspace) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || T <= 0 || Hs <= 0 || Ws <= 0 || d <= 0 || block <= 0 || tt <= 0 ||
      th <= 0 || tw <= 0)
    return BSA_ERR_INVALID_ARG;
  if (int64_t(B) * H >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  const int BH = B * H;
  const int hc = heads_per_chunk > 0 ? (heads_per_chunk < BH ? heads_per_chunk : BH)
                                     : default_chunk(BH);
  const int64_t n = int64_t(T) * Hs * Ws;
  const int64_t n_pad = (n + block - 1) / block * block;
  if (n_pad >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  const int nb = int(n_pad / block);
  const int words = (nb + 31) / 32;
  if (workspace_bytes < bsa_attention_host_workspace(B, H, T, Hs, Ws, d, block, heads_per_chunk))
    return BSA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BSA_ERR_MISALIGNED;
  DeviceCtx* ctx = device_ctx();
  if (!ctx) return BSA_ERR_LAUNCH;

  cudaStream_t comp = static_cast<cudaStream_t>(stream);
  // the copy streams start after everything already queued on the caller's
  // stream (an earlier call may still be using this workspace)
  if (cudaEventRecord(ctx->start, comp) != cudaSuccess ||
      cudaStreamWaitEvent(ctx->copy_in, ctx->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(ctx->copy_out, ctx->start, 0) != cudaSuccess)
    return BSA_ERR_LAUNCH;

  const SlotLayout L = slot_layout(hc, n, n_pad, d, nb);
  char* ws = static_cast<char*>(workspace);
  const size_t head_frame = size_t(n) * d * 2, head_mask = size_t(nb) * nb;
  const size_t head_lse = size_t(n_pad) * 4;
  // Chunk boundaries: with room for it, the first and the last chunk hold one
  // head each, so that the pipeline fills (the first copy-in before any
  // kernel) and drains (the last kernels and copy-out after the last copy-in)
  // in one head's time; the chunks between hold hc heads.
  std::vector<int> start{0};
  if (hc > 1 && BH > 2) {
    start.push_back(1);
    for (int h = 1 + hc; h < BH - 1; h += hc) start.push_back(h);
    start.push_back(BH - 1);
  } else {
    for (int h = hc; h < BH; h += hc) start.push_back(h);
  }
  start.push_back(BH);
  const int chunks = int(start.size()) - 1;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  for (int c = 0; c < chunks; ++c) {
    const int s = c % kSlots;
    char* base = ws + size_t(s) * L.bytes;
    const int h0 = start[c], hn = start[c + 1] - start[c];
    // ---- copy in (waits until chunk c - 2 has finished reading this slot)
    if (c >= kSlots && !ok(cudaStreamWaitEvent(ctx->copy_in, ctx->comp_done[s], 0)))
      return BSA_ERR_LAUNCH;
    const void* src[3] = {q, k, v};
    const size_t dst[3] = {L.qf, L.kf, L.vf};
    for (int i = 0; i < 3; ++i)
      if (!ok(cudaMemcpyAsync(base + dst[i], static_cast<const char*>(src[i]) + h0 * head_frame,
                              hn * head_frame, cudaMemcpyHostToDevice, ctx->copy_in)))
        return BSA_ERR_LAUNCH;
    if (!ok(cudaMemcpyAsync(base + L.dense, mask + h0 * head_mask, hn * head_mask,
                            cudaMemcpyHostToDevice, ctx->copy_in)) ||
        !ok(cudaEventRecord(ctx->h2d_done[s], ctx->copy_in)))
      return BSA_ERR_LAUNCH;
    // ---- compute (waits for its inputs, and for chunk c - 2's outputs to leave)
    if (!ok(cudaStreamWaitEvent(comp, ctx->h2d_done[s], 0))) return BSA_ERR_LAUNCH;
    if (c >= kSlots && !ok(cudaStreamWaitEvent(comp, ctx->d2h_done[s], 0))) return BSA_ERR_LAUNCH;
    auto p32 = [&](size_t off) { return reinterpret_cast<int32_t*>(base + off); };
    bsa_status st = bsa_pack_mask(reinterpret_cast<const uint8_t*>(base + L.dense), 1, hn, nb, nb,
                                  reinterpret_cast<uint32_t*>(base + L.bits), p32(L.counts),
                                  p32(L.offsets), nullptr, p32(L.schedule), base + L.pack_ws,
                                  L.pack_ws_bytes, comp);
    for (int i = 0; i < 3 && st == BSA_OK; ++i)
      st = bsa_tile_permute(base + dst[i], base + (i == 0 ? L.qp : i == 1 ? L.kp : L.vp), 1, hn, T,
                            Hs, Ws, d, tt, th, tw, int(n_pad), comp);
    if (st != BSA_OK) return st;
    bsa_mask m;
    m.bits = reinterpret_cast<const uint32_t*>(base + L.bits);
    m.counts = p32(L.counts);
    m.row_offsets = p32(L.offsets);
    m.col_idx = nullptr;
    m.schedule = p32(L.schedule);
    m.B = 1;
    m.H = hn;
    m.nb_q = nb;
    m.nb_k = nb;
    m.words = words;
    st = bsa_forward(base + L.qp, base + L.kp, base + L.vp, &m, base + L.op,
                     reinterpret_cast<float*>(base + L.lse), 1, hn, int(n), int(n_pad), d, block,
                     softmax_scale, comp);
    if (st == BSA_OK)
      st = bsa_tile_unpermute(base + L.op, base + L.of, 1, hn, T, Hs, Ws, d, tt, th, tw,
                              int(n_pad), comp);
    if (st != BSA_OK) return st;
    if (!ok(cudaEventRecord(ctx->comp_done[s], comp))) return BSA_ERR_LAUNCH;
    // ---- copy out
    if (!ok(cudaStreamWaitEvent(ctx->copy_out, ctx->comp_done[s], 0)) ||
        !ok(cudaMemcpyAsync(static_cast<char*>(out) + h0 * head_frame, base + L.of,
                            hn * head_frame, cudaMemcpyDeviceToHost, ctx->copy_out)) ||
        !ok(cudaMemcpyAsync(reinterpret_cast<char*>(lse) + h0 * head_lse, base + L.lse,
                            hn * head_lse, cudaMemcpyDeviceToHost, ctx->copy_out)) ||
        !ok(cudaEventRecord(ctx->d2h_done[s], ctx->copy_out)))
      return BSA_ERR_LAUNCH;
  }
  // join: the caller's stream waits for the last copy-out of each slot
  for (int s = 0; s < kSlots && s < chunks; ++s)
    if (!ok(cudaStreamWaitEvent(comp, ctx->d2h_done[s], 0))) return BSA_ERR_LAUNCH;
  return BSA_OK;
}
