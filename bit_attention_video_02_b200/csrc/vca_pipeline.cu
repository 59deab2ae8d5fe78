// vca_pipeline.cu -- the whole path from host buffers to host buffers, with the
// host<->device copies overlapped with the kernels.
//
// A layer's (batch, head) units are independent ("VC-Attention: Training-Free
// Low-Bit Attention Speeds Video Diffusion Up to 3.6x": grouping, quantisation
// and attention are all per head), so the layer is cut into chunks of heads and
// run as a three-stage pipeline over two device slots: copy chunk c+1 in while
// chunk c is grouped, quantised and attended, and copy chunk c-1's output out.
// A slot's Q, K and V are dead once the quantiser has read them, so the next
// input copy into that slot waits only for that, and the attention that
// rewrites its O waits for the output copy.
// Each chunk runs exactly the per-head kernels of vca_cluster_permute,
// vca_smooth_quantize_qkv and vca_attention_fwd, so the result is the same, bit
// for bit, as running the three calls on the whole layer.
#include <mutex>
#include <vector>

#include "vca_host.h"

using namespace vca;

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Byte layout of one device slot for a chunk of `u` (batch, head) units.
struct Slot {
  size_t q, k, v, o, cent, assign, perm, qq, kq, vrt, qs, ks, ve, vm, ws, total;
};

Slot slot_layout(int u, int N, int d, int k) {
  const int nb = (N + 127) / 128;
  const size_t Np = (size_t)nb * 128, un = (size_t)u * N;
  Slot s;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  s.q = take(un * d * 2);
  s.k = take(un * d * 2);
  s.v = take(un * d * 2);
  s.o = take(un * d * 2);
  s.cent = take((size_t)u * k * d * 4);
  s.assign = take(un * 4);
  s.perm = take(un * 4);
  s.qq = take((size_t)u * Np * d);
  s.kq = take((size_t)u * Np * d);
  s.vrt = take((size_t)u * Np * d);
  s.qs = take((size_t)u * nb * 4);
  s.ks = take((size_t)u * nb * 4);
  s.ve = take((size_t)u * nb);
  s.vm = take((size_t)u * nb * d * 2);
  size_t ws = vca_cluster_permute_workspace_size(1, u, N, k);
  ws = ws > vca_smooth_quantize_workspace_size(1, u, N) ? ws : vca_smooth_quantize_workspace_size(1, u, N);
  ws = ws > vca_attention_workspace_size(1, u, N) ? ws : vca_attention_workspace_size(1, u, N);
  s.ws = take(ws);
  s.total = off;
  return s;
}

// Three non-blocking streams per device, created on first use and kept for the
// life of the process.
struct Streams {
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
};
std::mutex g_streams_mu;
Streams g_streams[64];

int get_streams(Streams* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(VCA_ERR_CUDA, "vca_vc_attention_host: no current device");
  std::lock_guard<std::mutex> lock(g_streams_mu);
  Streams& s = g_streams[dev];
  if (!s.h2d) {
    if (cudaStreamCreateWithFlags(&s.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&s.comp, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&s.d2h, cudaStreamNonBlocking) != cudaSuccess)
      return fail(VCA_ERR_CUDA, "vca_vc_attention_host: cannot create streams");
  }
  *out = s;
  return VCA_OK;
}

// Chunk boundaries.  A chunk of s units takes about 0.8 s units' compute time to
// copy in while the output copy runs the other way (B200 over PCIe: ≈ 1.3 ms per
// Wan-shaped head in, ≈ 1.7 ms of kernels), so the sizes grow by 1.5x from one
// unit up to `u`: each chunk's input copy then fits under the previous chunk's
// compute while the pipeline fills.  The last two chunks hold 3 units and 1
// unit, so the output copy that nothing overlaps is one unit's and the one
// before it fits under that unit's compute.  The units between are split
// evenly into chunks of at most u.  starts[i] is the first unit of chunk i,
// starts.back() == units.
std::vector<int> chunk_starts(int units, int u) {
  std::vector<int> head, tail, sizes;
  int used = 0;
  for (int s = 1; s < u && used + s <= units; s = (3 * s + 1) / 2 < u ? (3 * s + 1) / 2 : u) {
    head.push_back(s);
    used += s;
  }
  for (int t : {1, 3}) {
    const int s = t < u ? t : u;
    if (used + s > units) break;
    tail.push_back(s);
    used += s;
  }
  const int rest = units - used;
  sizes = head;
  if (rest > 0) {
    const int nm = (rest + u - 1) / u, base = rest / nm, extra = rest % nm;
    for (int i = 0; i < nm; ++i) sizes.push_back(base + (i < extra ? 1 : 0));
  }
  sizes.insert(sizes.end(), tail.rbegin(), tail.rend());
  std::vector<int> starts;
  int pos = 0;
  for (int s : sizes) {
    starts.push_back(pos);
    pos += s;
  }
  starts.push_back(units);
  return starts;
}

// The nine events of one call (start, and per slot: input landed, input read
// by the quantiser, compute done, output copied), destroyed on every return
// path.
struct Events {
  cudaEvent_t e[9] = {};
  bool create() {
    for (cudaEvent_t& x : e)
      if (cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
  ~Events() {
    for (cudaEvent_t x : e)
      if (x) cudaEventDestroy(x);
  }
};

int units_per_chunk(int units, int heads_per_chunk) {
  if (heads_per_chunk > 0) return heads_per_chunk < units ? heads_per_chunk : units;
  const int u = (units + 3) / 4;   // about four chunks at full size, between the ramps
  return u < 1 ? 1 : u;
}

}  // namespace

extern "C" size_t vca_vc_attention_host_buffer_size(int B, int H, int N, int d, int k, int heads_per_chunk) {
  if (B < 1 || H < 1 || N < 1 || d != VCA_HEAD_DIM || k < 1 || k > VCA_MAX_CLUSTERS) return 0;
  const int u = units_per_chunk(B * H, heads_per_chunk);
  return 2 * slot_layout(u, N, d, k).total;
}

extern "C" int vca_vc_attention_host(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H, int N,
                                     int d, int k, int iters, float softmax_scale, vca_bf16* O, int heads_per_chunk,
                                     void* dev_buf, size_t dev_bytes, vca_stream_t stream) {
  const char* fn = "vca_vc_attention_host";
  if (!Q || !K || !V || !O || !dev_buf) return fail(VCA_ERR_INVALID, "%s: null pointer", fn);
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "%s: d must be 128", fn);
  if (B < 1 || H < 1 || N < 1 || k < 1 || k > VCA_MAX_CLUSTERS || iters < 1)
    return fail(VCA_ERR_INVALID, "%s: bad shape or k-means arguments", fn);
  if (heads_per_chunk < 0) return fail(VCA_ERR_INVALID, "%s: heads_per_chunk must be >= 0", fn);
  const int units = B * H;
  const int u = units_per_chunk(units, heads_per_chunk);
  const Slot L = slot_layout(u, N, d, k);
  if (dev_bytes < 2 * L.total) return fail(VCA_ERR_WORKSPACE, "%s: device buffer too small", fn);
  Streams st;
  int rc = get_streams(&st);
  if (rc) return rc;

  // the pipeline starts after the work already queued on the caller's stream
  Events evs;
  if (!evs.create()) return fail(VCA_ERR_CUDA, "%s: cannot create events", fn);
  cudaEvent_t start = evs.e[0], *ev_in = evs.e + 1, *ev_read = evs.e + 3, *ev_done = evs.e + 5, *ev_free = evs.e + 7;
  cudaEventRecord(start, (cudaStream_t)stream);
  cudaStreamWaitEvent(st.h2d, start, 0);
  cudaStreamWaitEvent(st.comp, start, 0);
  cudaStreamWaitEvent(st.d2h, start, 0);

  const size_t row = (size_t)N * d;   // elements per unit
  char* base = (char*)dev_buf;
  const std::vector<int> starts = chunk_starts(units, u);
  const int nchunks = (int)starts.size() - 1;
  // each call starts with clean status words in both slots' workspaces
  for (int s = 0; s < 2 && !rc; ++s) rc = vca_reset_status(base + (size_t)s * L.total + L.ws, st.comp);
  for (int c = 0; c < nchunks && !rc; ++c) {
    const int s = c & 1;
    const int u0 = starts[c], uc = starts[c + 1] - u0;
    char* b = base + (size_t)s * L.total;
    const size_t bytes = (size_t)uc * row * 2;
    // slot s takes new inputs once chunk c-2's quantiser has read its Q, K, V
    // (attention reads only the codes), and a new output once chunk c-2's O
    // has left the device (below)
    if (c >= 2) cudaStreamWaitEvent(st.h2d, ev_read[s], 0);
    if (cudaMemcpyAsync(b + L.q, Q + (size_t)u0 * row, bytes, cudaMemcpyHostToDevice, st.h2d) != cudaSuccess ||
        cudaMemcpyAsync(b + L.k, K + (size_t)u0 * row, bytes, cudaMemcpyHostToDevice, st.h2d) != cudaSuccess ||
        cudaMemcpyAsync(b + L.v, V + (size_t)u0 * row, bytes, cudaMemcpyHostToDevice, st.h2d) != cudaSuccess) {
      rc = fail(VCA_ERR_CUDA, "%s: host-to-device copy failed", fn);
      break;
    }
    cudaEventRecord(ev_in[s], st.h2d);
    cudaStreamWaitEvent(st.comp, ev_in[s], 0);
    void* ws = b + L.ws;
    const size_t wsb = L.total - L.ws;
    vca_bf16* Vd = (vca_bf16*)(b + L.v);
    rc = vca_cluster_permute(Vd, 1, uc, N, d, k, iters, nullptr, (float*)(b + L.cent), (int32_t*)(b + L.assign),
                             (int32_t*)(b + L.perm), ws, wsb, st.comp);
    if (!rc)
      rc = vca_smooth_quantize_qkv((vca_bf16*)(b + L.q), (vca_bf16*)(b + L.k), Vd, (int32_t*)(b + L.perm), 1, uc,
                                   N, d, 128, (uint8_t*)(b + L.qq), (float*)(b + L.qs), (uint8_t*)(b + L.kq),
                                   (float*)(b + L.ks), (uint8_t*)(b + L.vrt), (int8_t*)(b + L.ve),
                                   (vca_bf16*)(b + L.vm), ws, wsb, st.comp);
    if (!rc) {
      cudaEventRecord(ev_read[s], st.comp);
      if (c >= 2) cudaStreamWaitEvent(st.comp, ev_free[s], 0);
      rc = vca_attention_fwd((uint8_t*)(b + L.qq), (float*)(b + L.qs), (uint8_t*)(b + L.kq), (float*)(b + L.ks),
                             (uint8_t*)(b + L.vrt), (int8_t*)(b + L.ve), (vca_bf16*)(b + L.vm), 1, uc, N, d,
                             softmax_scale, (vca_bf16*)(b + L.o), nullptr, ws, wsb, st.comp);
    }
    if (rc) break;
    cudaEventRecord(ev_done[s], st.comp);
    cudaStreamWaitEvent(st.d2h, ev_done[s], 0);
    if (cudaMemcpyAsync(O + (size_t)u0 * row, b + L.o, bytes, cudaMemcpyDeviceToHost, st.d2h) != cudaSuccess) {
      rc = fail(VCA_ERR_CUDA, "%s: device-to-host copy failed", fn);
      break;
    }
    cudaEventRecord(ev_free[s], st.d2h);
  }
  // blocking call: everything queued above has finished when it returns
  const bool sync_ok = cudaStreamSynchronize(st.h2d) == cudaSuccess &&
                       cudaStreamSynchronize(st.comp) == cudaSuccess &&
                       cudaStreamSynchronize(st.d2h) == cudaSuccess;
  if (rc) return rc;
  if (!sync_ok) return fail(VCA_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(cudaGetLastError()));
  // device-side errors of either slot (timeouts, non-finite inputs)
  for (int s = 0; s < 2 && s < nchunks; ++s) {
    int where = 0, info = 0;
    rc = vca_check_status(base + (size_t)s * L.total + L.ws, nullptr, &where, &info);
    if (rc) return rc;
  }
  return VCA_OK;
}
