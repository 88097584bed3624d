// C ABI of the MoE layer forward (declared in include/moe.h): argument validation,
// workspace layout, stage orchestration on one stream, device status word and tracing.
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {

// ------------------------------------------------------------------ device properties
int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_DISABLE_PDL");
    return v == nullptr || v[0] == '\0' || std::strcmp(v, "0") == 0;
  }();
  return on;
}

// ------------------------------------------------------------------ side stream
// The shared expert needs only x, so for decode-sized batches (T*K <= kOverlapMaxPairs)
// moe_layer_forward runs it on a second stream of the library's own, next to the
// permutation kernels of the caller's stream: those are latency-bound there and fit on
// the SMs beside the shared expert's GEMM CTAs (measured on B200: DeepSeek-V3 shapes at
// T=128, 1.95 ms per layer against 2.01 ms on one stream).  At prefill sizes the layer is
// held by the power cap and the overlap bought nothing (7.90 against 7.89 ms at T=8192),
// so it stays on one stream.  One
// non-blocking stream and two events per device, made on first use and kept until exit
// (no device memory).  The work is forked from and joined back into the caller's stream
// with events, so stream order, and CUDA graph capture of the caller's stream, see the
// same dependencies as a single-stream layer.  Layers on one device share the side
// stream: their shared-expert GEMMs run one after the other.
namespace {
struct Side {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
Side g_side[64];

constexpr long long kOverlapMaxPairs = 16384;

bool overlap_shared_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_SERIAL_SHARED_EXPERT");
    return v == nullptr || v[0] == '\0' || std::strcmp(v, "0") == 0;
  }();
  return on;
}

// The side stream of the current device, or nullptr (then everything stays on one stream).
const Side* side_for_current_device() {
  if (!overlap_shared_enabled()) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_side_mu);
  Side& sd = g_side[dev];
  if (sd.stream == nullptr) {
    cudaStream_t s = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamDestroy(s);
      if (f) cudaEventDestroy(f);
      return nullptr;
    }
    sd.stream = s;
    sd.fork = f;
    sd.join = j;
  }
  return &sd;
}
}  // namespace

// ------------------------------------------------------------------ copy streams
// moe_layer_forward_host_batches copies activations in on one stream and outputs out on
// another, both the library's own (non-blocking, made on first use per device and kept
// until exit), ordered against the layer's kernels on the caller's stream by events: per
// staging slot, `in` (activations landed), `done` (the layer has read them and written its
// output) and `out` (the output has left the slot).
namespace {
struct Copies {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t landed[2] = {nullptr, nullptr}, done[2] = {nullptr, nullptr}, left[2] = {nullptr, nullptr};
};
std::mutex g_copy_mu;  // held while a call enqueues, so calls' event records do not interleave
Copies g_copies[64];

const Copies* copies_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  Copies& c = g_copies[dev];
  if (c.in != nullptr) return &c;
  Copies n;
  bool ok = cudaStreamCreateWithFlags(&n.in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&n.out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming) == cudaSuccess;
  for (int s = 0; s < 2 && ok; ++s)
    ok = cudaEventCreateWithFlags(&n.landed[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&n.done[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&n.left[s], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    if (n.in) cudaStreamDestroy(n.in);
    if (n.out) cudaStreamDestroy(n.out);
    for (cudaEvent_t e : {n.fork, n.landed[0], n.landed[1], n.done[0], n.done[1], n.left[0], n.left[1]})
      if (e) cudaEventDestroy(e);
    return nullptr;
  }
  c = n;
  return &c;
}
}  // namespace

// ------------------------------------------------------------------ tracing
namespace {
struct Trace {
  bool on = false;
  uint32_t mask = 0;
  int cap = 0;
  int n = 0;
  bool open = false;
  std::vector<cudaEvent_t> ev;
  std::vector<int> kid;
};
Trace g_trace;
}  // namespace

void trace_before(int kid, cudaStream_t st) {
  Trace& t = g_trace;
  t.open = false;
  if (!t.on || !((t.mask >> kid) & 1u) || t.n >= t.cap) return;
  if (cudaEventRecord(t.ev[2 * t.n], st) == cudaSuccess) t.open = true;
}

void trace_after(int kid, cudaStream_t st) {
  Trace& t = g_trace;
  if (!t.open) return;
  t.open = false;
  if (cudaEventRecord(t.ev[2 * t.n + 1], st) == cudaSuccess) {
    t.kid[t.n] = kid;
    ++t.n;
  }
}

// ------------------------------------------------------------------ workspace layout
namespace {

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  size_t status, logits, xb, ids, w, counts, offsets, sched, counter, row_of_pair, pair_of_row, chunk_counts;
  size_t x_perm, x_perm_scale, h, y_perm, h_sh, y_sh, total;
  size_t x_atoms, h_atoms, wg_atoms, wu_atoms, wd_atoms;
  size_t x_stage[2], x_scale_stage[2], out_stage[2], total_host;
  long long max_rows;
};

// e4m3 activations (with e4m3 or e2m1 expert weights)
bool is_fp8(const moe_params_t* p) { return p->dtype == MOE_DTYPE_FP8_E4M3 || p->dtype == MOE_DTYPE_FP8_FP4; }
// e2m1 expert weights whose scale atoms the caller prepared (moe_prepare_fp4_scales)
bool is_fp4(const moe_params_t* p) { return p->dtype == MOE_DTYPE_FP8_FP4; }

// Bucket alignment: 128 rows (one-SM GEMM tiles) unless the caller asks for 256 (two-SM
// cta_group::2 tiles).  Measured on B200, the pair tiles' third less SM-side traffic did
// not pay for the extra pad rows that 256-row buckets add (about 6% more MMA work on the
// Mixtral and FP8 skew shapes), so they are opt-in.
int block_m_of(const moe_params_t* p) { return p->block_m != 0 ? p->block_m : kBlockM; }

Layout layout(const moe_params_t* p) {
  Layout L{};
  const long long T = p->T, H = p->H, I = p->I, E = p->E, K = p->K;
  const long long P = T * K;
  const long long bm = block_m_of(p);
  const long long rows = p->masked_cap > 0 ? E * p->masked_cap : P + E * (bm - 1);
  const long long rows_t = (rows + kBlockM2 - 1) / kBlockM2 * kBlockM2;  // whole M-tile pairs
  const long long nchunks = (P + kPermChunk - 1) / kPermChunk;
  const size_t xelem = is_fp8(p) ? 1 : 2;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o += up(bytes); return at; };
  L.max_rows = rows;
  L.status = take(256);
  L.logits = take(router_k_splits(T, p->H, p->E) * T * E * 4);  // one [T,E] slice per K-slice
  L.xb = take(is_fp8(p) ? T * H * 2 : 0);
  L.ids = take(P * 4);
  L.w = take(P * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.sched = take(p->masked_cap > 0 ? (E + 1) * 4 : 0);
  L.counter = take(8);  // work counters of the two-tile gate/up and down kernels
  L.row_of_pair = take(P * 4);
  L.pair_of_row = take(rows * 4);
  L.chunk_counts = take((nchunks > 0 ? nchunks : 1) * E * 4);
  L.x_perm = take(rows * H * xelem);
  L.x_perm_scale = take(is_fp8(p) ? rows * (H / 128) * 4 : 0);
  L.h = take(rows_t * I * 2);
  L.y_perm = take(rows * H * 4);
  L.h_sh = take(T * static_cast<long long>(p->I_shared) * 2);
  L.y_sh = take(p->I_shared > 0 || p->fused_combine ? T * H * 4 : 0);  // also the fused-combine accumulator
  const bool f8 = is_fp8(p);
  const bool w8 = p->dtype == MOE_DTYPE_FP8_E4M3;  // e4m3 weights: atoms built per call
  // e4m3 scale atoms: 512 bytes per 128 rows and 4 K blocks of 128
  const long long hk4 = (H / 128 + 3) / 4, ik4 = (I / 128 + 3) / 4;
  L.x_atoms = take(f8 ? rows_t / 128 * hk4 * 512 : 0);
  L.h_atoms = take(f8 ? rows_t / 128 * ik4 * 512 : 0);
  L.wg_atoms = take(w8 ? E * (I / 128) * hk4 * 512 : 0);
  L.wu_atoms = take(w8 ? E * (I / 128) * hk4 * 512 : 0);
  L.wd_atoms = take(w8 ? E * (H / 128) * ik4 * 512 : 0);
  L.total = o;
  for (int slot = 0; slot < 2; ++slot) {  // host entry points: two device staging slots
    L.x_stage[slot] = take(T * H * xelem);
    L.x_scale_stage[slot] = take(is_fp8(p) ? T * (H / 128) * 4 : 0);
    L.out_stage[slot] = take(T * H * 2);
  }
  L.total_host = o;
  return L;
}

template <class Tp>
Tp* at(void* ws, size_t off) {
  return reinterpret_cast<Tp*>(static_cast<uint8_t*>(ws) + off);
}

moe_status_t validate(const moe_params_t* p) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (p->T < 0 || p->H <= 0 || p->I <= 0 || p->E <= 0 || p->K <= 0) return MOE_ERR_INVALID_ARG;
  if (p->E > kMaxExperts || p->K > kMaxTopK || p->K > p->E) return MOE_ERR_INVALID_ARG;
  if (p->score_fn != MOE_SCORE_SOFTMAX && p->score_fn != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (p->dtype != MOE_DTYPE_BF16 && p->dtype != MOE_DTYPE_FP8_E4M3 && p->dtype != MOE_DTYPE_FP8_FP4)
    return MOE_ERR_INVALID_ARG;
  if (p->n_group < 1 || p->n_group > 32 || p->E % p->n_group != 0) return MOE_ERR_INVALID_ARG;
  if (p->n_group > 1) {
    const int gs = p->E / p->n_group;
    if (p->topk_group < 1 || p->topk_group > p->n_group) return MOE_ERR_INVALID_ARG;
    if (p->group_topn < 1 || p->group_topn > gs) return MOE_ERR_INVALID_ARG;
    if (p->topk_group * gs < p->K) return MOE_ERR_INVALID_ARG;
  }
  if (p->I_shared < 0) return MOE_ERR_INVALID_ARG;
  if (p->H % 128 != 0 || p->I % 128 != 0 || p->I_shared % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (p->block_m != 0 && p->block_m != kBlockM && p->block_m != kBlockM2) return MOE_ERR_UNSUPPORTED;
  if (is_fp8(p) && p->I_shared > 0) return MOE_ERR_UNSUPPORTED;
  if (is_fp4(p) && p->block_m == kBlockM2) return MOE_ERR_UNSUPPORTED;
  if (p->fused_combine != 0 && p->fused_combine != 1) return MOE_ERR_INVALID_ARG;
  if (p->fused_combine && (p->dtype != MOE_DTYPE_BF16 || p->block_m == kBlockM2)) return MOE_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(p->T) * p->K + static_cast<long long>(p->E) * (kBlockM2 - 1);
  if (rows >= (1LL << 31) / 2) return MOE_ERR_INVALID_ARG;
  if (p->masked_cap < 0) return MOE_ERR_INVALID_ARG;
  if (p->masked_cap > 0) {
    if (p->masked_cap % kBlockM != 0 || p->block_m == kBlockM2) return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(p->E) * p->masked_cap >= (1LL << 31) / 2) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
bool aligned32(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 31u) == 0; }

// Weight scales as the FFN reads them: fp32 block scales (e4m3 weights) or prepared
// 512-byte atoms (e2m1 weights, read with 16-byte bulk copies).
bool weight_scales_ok(const moe_params_t* p, const void* g, const void* u, const void* d) {
  if (!is_fp8(p)) return true;
  if (!g || !u || !d) return false;
  return !is_fp4(p) || (aligned16(g) && aligned16(u) && aligned16(d));
}

moe_status_t check_ws(const moe_params_t* p, const void* ws, size_t ws_bytes, bool host) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_INVALID_ARG;
  const Layout L = layout(p);
  if (ws_bytes < (host ? L.total_host : L.total)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                          \
  do {                                         \
    const moe_status_t s_ = (expr);            \
    if (s_ != MOE_OK) return s_;               \
  } while (0)

#define MOE_CUDA(expr) MOE_TRY(cuda_status(expr))

// ---------------------------------------------------------------- stages (no validation)
moe_status_t do_route(const moe_params_t* p, const void* x, const float* x_scale, const void* w_r,
                      const float* bias, int32_t* ids, float* w, void* ws, cudaStream_t st) {
  const Layout L = layout(p);
  int32_t* status = at<int32_t>(ws, L.status);
  const void* xb = x;
  if (is_fp8(p)) {
    MOE_CUDA(launch_dequant_x(static_cast<const uint8_t*>(x), x_scale, p->T, p->H, at<void>(ws, L.xb), st));
    xb = at<void>(ws, L.xb);
  }
  float* logits = at<float>(ws, L.logits);
  MOE_CUDA(gemm_router(xb, w_r, p->T, p->H, p->E, logits, status, st));
  MOE_CUDA(launch_topk(logits, *p, bias, ids, w, st, router_k_splits(p->T, p->H, p->E)));
  return MOE_OK;
}

// fill_pad: zero x_perm's pad rows (moe_permute's contract); the layer skips it (its GEMMs
// never store a pad row).  x_atoms (FP8 layers, only with fill_pad false): the copy writes
// x's scales straight into the GEMM's scale atoms instead of x_perm_scale.
moe_status_t do_permute(const moe_params_t* p, const int32_t* ids, const void* x, const float* x_scale,
                        int32_t* counts, int32_t* offsets, int32_t* rop, int32_t* por, void* x_perm,
                        float* x_perm_scale, void* ws, cudaStream_t st, bool fill_pad = true,
                        uint8_t* x_atoms = nullptr) {
  const Layout L = layout(p);
  return cuda_status(launch_permute(*p, block_m_of(p), ids, x, x_scale, counts, offsets, rop, por, x_perm, x_perm_scale,
                                    at<int32_t>(ws, L.chunk_counts), at<int32_t>(ws, L.status), st, fill_pad,
                                    x_atoms));
}

moe_status_t do_expert_ffn_fp8(const moe_params_t* p, const void* x_perm, const float* x_perm_scale,
                               const int32_t* offsets, const int32_t* counts, const void* w_gate,
                               const void* w_up, const void* w_down, const void* wgs,
                               const void* wus, const void* wds, void* y_perm, void* ws,
                               cudaStream_t st, bool x_atoms_ready = false) {
  const Layout L = layout(p);
  int32_t* status = at<int32_t>(ws, L.status);
  // masked layout: the GEMMs walk a compact schedule and address expert e's rows at e*cap
  const int cap = p->masked_cap;
  const int32_t* sched = offsets;
  if (cap > 0) {
    MOE_CUDA(launch_masked_schedule(counts, p->E, at<int32_t>(ws, L.sched), st));
    sched = at<int32_t>(ws, L.sched);
  }
  // weight scale atoms: e2m1 weights bring theirs (prepared once); e4m3 weights' fp32
  // block scales are turned into atoms here
  const bool w4 = is_fp4(p);
  const uint8_t* wg_atoms = static_cast<const uint8_t*>(wgs);
  const uint8_t* wu_atoms = static_cast<const uint8_t*>(wus);
  const uint8_t* wd_atoms = static_cast<const uint8_t*>(wds);
  if (!w4) {
    const long long rows_gu = static_cast<long long>(p->E) * (p->I / 128);   // 128-row weight blocks
    const long long rows_d = static_cast<long long>(p->E) * (p->H / 128);
    MOE_CUDA(launch_sf_blocks_to_atoms(static_cast<const float*>(wgs), rows_gu, p->H / 128,
                                       at<uint8_t>(ws, L.wg_atoms), st));
    MOE_CUDA(launch_sf_blocks_to_atoms(static_cast<const float*>(wus), rows_gu, p->H / 128,
                                       at<uint8_t>(ws, L.wu_atoms), st));
    MOE_CUDA(launch_sf_blocks_to_atoms(static_cast<const float*>(wds), rows_d, p->I / 128,
                                       at<uint8_t>(ws, L.wd_atoms), st));
    wg_atoms = at<uint8_t>(ws, L.wg_atoms);
    wu_atoms = at<uint8_t>(ws, L.wu_atoms);
    wd_atoms = at<uint8_t>(ws, L.wd_atoms);
  }
  if (!x_atoms_ready)
    MOE_CUDA(launch_sf_rows_to_atoms(x_perm_scale, p->H / 128, offsets, p->E, L.max_rows,
                                     at<uint8_t>(ws, L.x_atoms), st));
  void* h = at<void>(ws, L.h);
  if (block_m_of(p) == kBlockM2) {
    MOE_CUDA(gemm_pair_gateup_swiglu_fp8(x_perm, at<uint8_t>(ws, L.x_atoms), L.max_rows, offsets, counts, p->E,
                                         w_gate, w_up, wg_atoms, wu_atoms,
                                         p->I, p->H, h, at<uint8_t>(ws, L.h_atoms), status, st));
    MOE_CUDA(gemm_pair_down_fp8(h, at<uint8_t>(ws, L.h_atoms), L.max_rows, offsets, counts, p->E, w_down,
                                wd_atoms, p->H, p->I, y_perm, status, st));
    return MOE_OK;
  }
  MOE_CUDA(gemm_gateup_swiglu_fp8(x_perm, at<uint8_t>(ws, L.x_atoms), L.max_rows, sched, counts, p->E,
                                  w_gate, w_up, wg_atoms, wu_atoms, p->I, p->H, h, at<uint8_t>(ws, L.h_atoms),
                                  status, st, cap, w4));
  MOE_CUDA(gemm_down_fp8(h, at<uint8_t>(ws, L.h_atoms), L.max_rows, sched, counts, p->E, w_down, wd_atoms,
                         p->H, p->I, y_perm, status, st, cap, w4));
  return MOE_OK;
}

// Gate/up with SwiGLU of the routed experts.  When the average expert holds at least two
// 128-row M-tiles (T*K >= 256*E) the two-tile kernel runs: one staged weight tile feeds the
// MMAs of two M-tiles (measured on B200: DeepSeek-V3 prefill gate/up 3.92 against 4.12 ms,
// Mixtral prefill 1.51 against 1.63 ms); at decode sizes almost every expert has one
// M-tile and the one-tile kernel is faster (1.22 against 1.27 ms).
bool two_tile_items(const moe_params_t* p, const int32_t* counts) {
  return counts != nullptr && p->E <= 1024 && static_cast<long long>(p->T) * p->K >= 256LL * p->E;
}

moe_status_t do_gateup(const moe_params_t* p, const void* x_perm, const int32_t* sched, const int32_t* counts,
                       const void* w_gate, const void* w_up, void* ws, cudaStream_t st,
                       const DualExtra* extra = nullptr) {
  const Layout L = layout(p);
  int32_t* status = at<int32_t>(ws, L.status);
  void* h = at<void>(ws, L.h);
  if (two_tile_items(p, counts))
    return cuda_status(gemm_gateup_swiglu_dual(x_perm, L.max_rows, sched, counts, p->E, w_gate, w_up, p->I, p->H,
                                               h, at<int32_t>(ws, L.counter), status, st, p->masked_cap,
                                               MOE_K_GATEUP, extra));
  return cuda_status(gemm_gateup_swiglu(x_perm, L.max_rows, sched, counts, p->E, 0, w_gate, w_up, p->I, p->H, h,
                                        status, MOE_K_GATEUP, st, p->masked_cap));
}

// Inside moe_layer_forward, y_perm is fp16 wherever the two-tile down projection runs (bf16
// layers at prefill sizes): half the bytes of fp32 for the down projection to write and the
// combine to read (measured on B200, DeepSeek-V3 prefill: down 1.90 against 2.05 ms, combine
// 0.23 against 0.36 ms, layer 7.13 against 7.46 ms), at 2^-11 relative rounding per element.
// An output beyond fp16's range (|y| > 65504) sets MOE_DEV_RANGE.  The stage entry points
// (moe_expert_ffn, moe_combine) keep fp32 y_perm.
bool layer_y16(const moe_params_t* p, const int32_t* counts) {
  return two_tile_items(p, counts) && p->H % 256 == 0 && !is_fp8(p);
}

// The shared expert of a bf16 layer on one stream (prefill sizes: its T rows hold at least
// two M-tiles) runs through the two-tile kernels as one dense group, y_sh in fp16.
bool shared_two_tile(const moe_params_t* p) {
  return !is_fp8(p) && p->T >= 256 && p->H % 256 == 0 && p->I_shared % 128 == 0;
}

// ... and when the routed experts run through the two-tile kernels too, it is one more group
// of their launches (one launch and one tail per projection instead of two).  Decided from
// the parameters alone (the side stream takes the shared expert for few pairs).
bool shared_merged(const moe_params_t* p) {
  const long long P = static_cast<long long>(p->T) * p->K;
  const bool side = P <= kOverlapMaxPairs && overlap_shared_enabled();
  return p->I_shared > 0 && !side && !p->fused_combine && shared_two_tile(p) && block_m_of(p) != kBlockM2 &&
         p->E <= 1024 && P >= 256LL * p->E;
}

// gu_extra / dn_extra: the shared expert as an extra group of the two-tile launches (only
// passed when those run, see shared_merged).
moe_status_t do_expert_ffn(const moe_params_t* p, const void* x_perm, const int32_t* offsets,
                           const int32_t* counts, const void* w_gate, const void* w_up,
                           const void* w_down, float* y_perm, void* ws, cudaStream_t st, bool y16 = false,
                           const DualExtra* gu_extra = nullptr, const DualExtra* dn_extra = nullptr) {
  const Layout L = layout(p);
  int32_t* status = at<int32_t>(ws, L.status);
  void* h = at<void>(ws, L.h);
  if (block_m_of(p) == kBlockM2) {
    MOE_CUDA(gemm_pair_gateup_swiglu(x_perm, L.max_rows, offsets, counts, p->E, w_gate, w_up, p->I, p->H, h,
                                     status, st));
    MOE_CUDA(gemm_pair_down(h, L.max_rows, offsets, counts, p->E, w_down, p->H, p->I, y_perm, status, st));
    return MOE_OK;
  }
  const int cap = p->masked_cap;
  const int32_t* sched = offsets;
  if (cap > 0) {  // masked layout: compact schedule, expert e's rows at e*cap
    MOE_CUDA(launch_masked_schedule(counts, p->E, at<int32_t>(ws, L.sched), st));
    sched = at<int32_t>(ws, L.sched);
  }
  MOE_TRY(do_gateup(p, x_perm, sched, counts, w_gate, w_up, ws, st, gu_extra));
  // the down projection takes two M-tiles per item under the same rule as gate/up
  // (measured: Mixtral prefill down 0.72 against 0.82 ms, DeepSeek-V3 prefill step 7.9
  // against 8.1 ms); its weight tiles are 256 rows, so H must be a multiple of 256
  if (two_tile_items(p, counts) && p->H % 256 == 0)
    MOE_CUDA(gemm_down_dual(h, L.max_rows, sched, counts, p->E, w_down, p->H, p->I, y_perm,
                            at<int32_t>(ws, L.counter) + 1, status, st, cap, y16, MOE_K_DOWN, dn_extra));
  else
    MOE_CUDA(gemm_down(h, L.max_rows, sched, counts, p->E, 0, w_down, p->H, p->I, y_perm, status,
                       MOE_K_DOWN, st, cap));
  return MOE_OK;
}

moe_status_t do_shared(const moe_params_t* p, const void* x, const void* wsg, const void* wsu,
                       const void* wsd, float* y_sh, void* ws, cudaStream_t st) {
  const Layout L = layout(p);
  int32_t* status = at<int32_t>(ws, L.status);
  void* h = at<void>(ws, L.h_sh);
  MOE_CUDA(gemm_gateup_swiglu(x, p->T, nullptr, nullptr, 1, p->T, wsg, wsu, p->I_shared, p->H, h,
                              status, MOE_K_SHARED_GATEUP, st));
  MOE_CUDA(gemm_down(h, p->T, nullptr, nullptr, 1, p->T, wsd, p->H, p->I_shared, y_sh, status,
                     MOE_K_SHARED_DOWN, st));
  return MOE_OK;
}

moe_status_t do_layer_after_fork(const moe_params_t* p, const void* x, const float* x_scale, const void* w_gate,
                                 const void* w_up, const void* w_down, const void* wgs, const void* wus,
                                 const void* wds, const void* wsg, const void* wsu, const void* wsd, void* out,
                                 int32_t* ids, float* w, int32_t* counts, float* y_sh, const Side* side, void* ws,
                                 cudaStream_t st);

moe_status_t do_layer(const moe_params_t* p, const void* x, const float* x_scale, const void* w_r,
                      const float* bias, const void* w_gate, const void* w_up, const void* w_down,
                      const void* wgs, const void* wus, const void* wds, const void* wsg,
                      const void* wsu, const void* wsd, void* out, int32_t* ids_out, float* w_out,
                      int32_t* counts_out, void* ws, cudaStream_t st) {
  const Layout L = layout(p);
  if (p->T == 0) return MOE_OK;
  int32_t* ids = ids_out ? ids_out : at<int32_t>(ws, L.ids);
  float* w = w_out ? w_out : at<float>(ws, L.w);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  MOE_TRY(do_route(p, x, x_scale, w_r, bias, ids, w, ws, st));
  // shared expert (y_sh, or the fused combine's accumulator): forked onto the side stream
  // here, joined back before its output is read
  const bool overlap = p->I_shared > 0 && static_cast<long long>(p->T) * p->K <= kOverlapMaxPairs;
  const Side* side = overlap ? side_for_current_device() : nullptr;
  float* y_sh = p->I_shared > 0 || p->fused_combine ? at<float>(ws, L.y_sh) : nullptr;
  if (side != nullptr) {
    // one host thread at a time between recording the fork and recording the join, so
    // another layer's records cannot come in between (a later join record only covers
    // more work of the side stream, so waiting on it stays correct)
    std::lock_guard<std::mutex> lock(g_side_mu);
    MOE_CUDA(cudaEventRecord(side->fork, st));
    MOE_CUDA(cudaStreamWaitEvent(side->stream, side->fork, 0));
    const moe_status_t s_sh = do_shared(p, x, wsg, wsu, wsd, y_sh, ws, side->stream);
    MOE_CUDA(cudaEventRecord(side->join, side->stream));
    if (s_sh != MOE_OK) {
      cudaStreamWaitEvent(st, side->join, 0);
      return s_sh;
    }
  }
  // from here on, every return first joins the side stream back into st
  const moe_status_t s_main = do_layer_after_fork(p, x, x_scale, w_gate, w_up, w_down, wgs, wus, wds, wsg, wsu,
                                                  wsd, out, ids, w, counts, y_sh, side, ws, st);
  if (s_main != MOE_OK && side != nullptr) cudaStreamWaitEvent(st, side->join, 0);
  return s_main;
}

moe_status_t do_layer_after_fork(const moe_params_t* p, const void* x, const float* x_scale, const void* w_gate,
                                 const void* w_up, const void* w_down, const void* wgs, const void* wus,
                                 const void* wds, const void* wsg, const void* wsu, const void* wsd, void* out,
                                 int32_t* ids, float* w, int32_t* counts, float* y_sh, const Side* side, void* ws,
                                 cudaStream_t st) {
  const Layout L = layout(p);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* rop = at<int32_t>(ws, L.row_of_pair);
  float* y_perm = at<float>(ws, L.y_perm);
  MOE_TRY(do_permute(p, ids, x, x_scale, counts, offsets, rop, at<int32_t>(ws, L.pair_of_row),
                     at<void>(ws, L.x_perm), at<float>(ws, L.x_perm_scale), ws, st, /*fill_pad=*/false,
                     is_fp8(p) ? at<uint8_t>(ws, L.x_atoms) : nullptr));
  if (p->fused_combine) {
    // acc starts as the shared expert's output (or zero); the routed down projection adds
    // w * y of every pair into it; one pass rounds it to bf16
    float* acc = y_sh;
    if (side == nullptr) {
      if (p->I_shared > 0) MOE_TRY(do_shared(p, x, wsg, wsu, wsd, acc, ws, st));
      else MOE_CUDA(cudaMemsetAsync(acc, 0, static_cast<size_t>(p->T) * p->H * sizeof(float), st));
    }
    int32_t* status = at<int32_t>(ws, L.status);
    void* h = at<void>(ws, L.h);
    const int cap = p->masked_cap;
    const int32_t* sched = offsets;
    if (cap > 0) {
      MOE_CUDA(launch_masked_schedule(counts, p->E, at<int32_t>(ws, L.sched), st));
      sched = at<int32_t>(ws, L.sched);
    }
    MOE_TRY(do_gateup(p, at<void>(ws, L.x_perm), sched, counts, w_gate, w_up, ws, st));
    if (side != nullptr) MOE_CUDA(cudaStreamWaitEvent(st, side->join, 0));  // acc holds y_sh
    MOE_CUDA(gemm_down_combine(h, L.max_rows, sched, counts, p->E, w_down, p->H, p->I,
                               at<int32_t>(ws, L.pair_of_row), w, p->K, acc, status, st, cap));
    return cuda_status(launch_f32_to_bf16(acc, static_cast<long long>(p->T) * p->H, out, st));
  }
  const bool merged = side == nullptr && shared_merged(p);
  if (is_fp8(p)) {
    MOE_TRY(do_expert_ffn_fp8(p, at<void>(ws, L.x_perm), at<float>(ws, L.x_perm_scale), offsets, counts,
                              w_gate, w_up, w_down, wgs, wus, wds, y_perm, ws, st, /*x_atoms_ready=*/true));
  } else if (merged) {
    // the shared expert as the extra group of the routed two-tile launches, y_sh in fp16
    const DualExtra gu{x, p->T, wsg, wsu, p->I_shared, p->H, at<void>(ws, L.h_sh)};
    const DualExtra dn{at<void>(ws, L.h_sh), p->T, wsd, nullptr, p->H, p->I_shared, y_sh};
    MOE_TRY(do_expert_ffn(p, at<void>(ws, L.x_perm), offsets, counts, w_gate, w_up, w_down, y_perm, ws, st,
                          layer_y16(p, counts), &gu, &dn));
  } else {
    MOE_TRY(do_expert_ffn(p, at<void>(ws, L.x_perm), offsets, counts, w_gate, w_up, w_down, y_perm, ws, st,
                          layer_y16(p, counts)));
  }
  bool ysh16 = merged;
  if (side != nullptr) {
    MOE_CUDA(cudaStreamWaitEvent(st, side->join, 0));
  } else if (merged) {
    // done inside the routed launches
  } else if (p->I_shared > 0 && shared_two_tile(p)) {
    // the dense shared expert at prefill sizes through the two-tile kernels, y_sh in fp16
    int32_t* status = at<int32_t>(ws, L.status);
    int32_t* ctr = at<int32_t>(ws, L.counter);
    MOE_CUDA(gemm_gateup_swiglu_dual(x, p->T, nullptr, nullptr, 1, wsg, wsu, p->I_shared, p->H,
                                     at<void>(ws, L.h_sh), ctr, status, st, 0, MOE_K_SHARED_GATEUP));
    MOE_CUDA(gemm_down_dual(at<void>(ws, L.h_sh), p->T, nullptr, nullptr, 1, wsd, p->H, p->I_shared, y_sh,
                            ctr + 1, status, st, 0, /*y_f16=*/true, MOE_K_SHARED_DOWN));
    ysh16 = true;
  } else if (p->I_shared > 0) {
    MOE_TRY(do_shared(p, x, wsg, wsu, wsd, y_sh, ws, st));
  }
  return cuda_status(launch_combine(*p, y_perm, rop, w, p->I_shared > 0 ? y_sh : nullptr, out, st,
                                    layer_y16(p, counts), ysh16));
}

moe_status_t check_layer_args(const moe_params_t* p, const void* x, const float* x_scale, const void* w_r,
                              const void* w_gate, const void* w_up, const void* w_down, const void* wsg,
                              const void* wsu, const void* wsd, const void* out) {
  if (!x || !w_r || !w_gate || !w_up || !w_down || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_r) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (is_fp8(p) && !x_scale) return MOE_ERR_INVALID_ARG;
  if (is_fp4(p) && !(aligned32(w_gate) && aligned32(w_up) && aligned32(w_down))) return MOE_ERR_INVALID_ARG;
  if (p->I_shared > 0) {
    if (!wsg || !wsu || !wsd) return MOE_ERR_INVALID_ARG;
    if (!aligned16(wsg) || !aligned16(wsu) || !aligned16(wsd)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_params_t* p) {
  if (validate(p) != MOE_OK) return 0;
  return layout(p).total;
}

size_t moe_workspace_size_host(const moe_params_t* p) {
  if (validate(p) != MOE_OK) return 0;
  return layout(p).total_host;
}

int32_t moe_effective_block_m(const moe_params_t* p) {
  if (validate(p) != MOE_OK) return -1;
  return block_m_of(p);
}

int64_t moe_max_padded_rows(const moe_params_t* p) {
  if (validate(p) != MOE_OK) return -1;
  return layout(p).max_rows;
}

moe_status_t moe_route(const moe_params_t* p, const void* x, const float* x_scale, const void* w_r,
                       const float* bias, int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes,
                       void* stream) {
  MOE_TRY(validate(p));
  MOE_TRY(check_ws(p, ws, ws_bytes, false));
  if (p->T == 0) return MOE_OK;  // empty batch: nothing to read or write
  if (!x || !w_r || !topk_ids || !topk_w || !aligned16(x) || !aligned16(w_r)) return MOE_ERR_INVALID_ARG;
  if (is_fp8(p) && !x_scale) return MOE_ERR_INVALID_ARG;
  return do_route(p, x, x_scale, w_r, bias, topk_ids, topk_w, ws, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_grouped_topk(const moe_params_t* p, const float* logits, const float* bias,
                              int32_t* topk_ids, float* topk_w, void* stream) {
  MOE_TRY(validate(p));
  if (p->T == 0) return MOE_OK;
  if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_topk(logits, *p, bias, topk_ids, topk_w, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_aux_free_bias_update(const int32_t* counts, int32_t E, float gamma, float* bias,
                                      void* stream) {
  if (!counts || !bias || E <= 0 || E > kMaxExperts) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_bias_update(counts, E, gamma, bias, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_permute(const moe_params_t* p, const int32_t* topk_ids, const void* x, const float* x_scale,
                         int32_t* counts, int32_t* offsets_padded, int32_t* row_of_pair, int32_t* pair_of_row,
                         void* x_perm, float* x_perm_scale, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(validate(p));
  MOE_TRY(check_ws(p, ws, ws_bytes, false));
  // an empty batch still writes counts (all 0), offsets and, masked, pair_of_row (all -1);
  // the [T,...] and [T*K] arrays are not touched and may be NULL
  const bool empty = p->T == 0;
  if ((!empty && (!topk_ids || !x || !row_of_pair)) || !counts || !offsets_padded || !pair_of_row || !x_perm)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  if (is_fp8(p) && ((!empty && !x_scale) || !x_perm_scale)) return MOE_ERR_INVALID_ARG;
  return do_permute(p, topk_ids, x, x_scale, counts, offsets_padded, row_of_pair, pair_of_row, x_perm,
                    x_perm_scale, ws, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_ffn(const moe_params_t* p, const void* x_perm, const float* x_perm_scale,
                            const int32_t* offsets_padded, const int32_t* counts, const void* w_gate,
                            const void* w_up, const void* w_down, const void* w_gate_scale,
                            const void* w_up_scale, const void* w_down_scale, void* y_perm,
                            void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(validate(p));
  MOE_TRY(check_ws(p, ws, ws_bytes, false));
  if (p->T == 0) return MOE_OK;
  if (!x_perm || !w_gate || !w_up || !w_down || !y_perm) return MOE_ERR_INVALID_ARG;
  if (p->masked_cap > 0 ? !counts : !offsets_padded) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  if (is_fp8(p) && !x_perm_scale) return MOE_ERR_INVALID_ARG;
  if (!weight_scales_ok(p, w_gate_scale, w_up_scale, w_down_scale)) return MOE_ERR_INVALID_ARG;
  if (is_fp4(p) && !(aligned32(w_gate) && aligned32(w_up) && aligned32(w_down))) return MOE_ERR_INVALID_ARG;
  if (offsets_padded == nullptr) {  // masked layout: expert e's rows start at e*cap
    const Layout L = layout(p);
    int32_t* offs = at<int32_t>(ws, L.offsets);
    MOE_CUDA(launch_masked_offsets(p->E, p->masked_cap, offs, static_cast<cudaStream_t>(stream)));
    offsets_padded = offs;
  }
  if (is_fp8(p))
    return do_expert_ffn_fp8(p, x_perm, x_perm_scale, offsets_padded, counts, w_gate, w_up, w_down,
                             w_gate_scale, w_up_scale, w_down_scale, y_perm, ws,
                             static_cast<cudaStream_t>(stream));
  return do_expert_ffn(p, x_perm, offsets_padded, counts, w_gate, w_up, w_down, static_cast<float*>(y_perm), ws,
                       static_cast<cudaStream_t>(stream));
}

moe_status_t moe_shared_expert_ffn(const moe_params_t* p, const void* x, const void* ws_gate,
                                   const void* ws_up, const void* ws_down, float* y_shared, void* ws,
                                   size_t ws_bytes, void* stream) {
  MOE_TRY(validate(p));
  MOE_TRY(check_ws(p, ws, ws_bytes, false));
  if (p->I_shared <= 0 || is_fp8(p)) return MOE_ERR_UNSUPPORTED;
  if (p->T == 0) return MOE_OK;
  if (!x || !ws_gate || !ws_up || !ws_down || !y_shared) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(ws_gate) || !aligned16(ws_up) || !aligned16(ws_down) || !aligned16(y_shared))
    return MOE_ERR_INVALID_ARG;
  return do_shared(p, x, ws_gate, ws_up, ws_down, y_shared, ws, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_combine(const moe_params_t* p, const void* y_perm, const int32_t* row_of_pair,
                         const float* topk_w, const float* y_shared, void* out, void* stream) {
  MOE_TRY(validate(p));
  if (p->T == 0) return MOE_OK;
  if (!y_perm || !row_of_pair || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(out) || (y_shared && !aligned16(y_shared))) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(*p, y_perm, row_of_pair, topk_w, y_shared, out,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_layer_forward(const moe_params_t* p, const void* x, const float* x_scale, const void* w_r,
                               const float* bias, const void* w_gate, const void* w_up, const void* w_down,
                               const void* w_gate_scale, const void* w_up_scale, const void* w_down_scale,
                               const void* ws_gate, const void* ws_up, const void* ws_down, void* out,
                               int32_t* topk_ids_out, float* topk_w_out, int32_t* counts_out, void* ws,
                               size_t ws_bytes, void* stream) {
  MOE_TRY(validate(p));
  MOE_TRY(check_ws(p, ws, ws_bytes, false));
  if (p->T == 0)  // empty batch: no pairs, so the only output is an all-zero counts_out
    return counts_out ? cuda_status(cudaMemsetAsync(counts_out, 0, static_cast<size_t>(p->E) * sizeof(int32_t),
                                                    static_cast<cudaStream_t>(stream)))
                      : MOE_OK;
  MOE_TRY(check_layer_args(p, x, x_scale, w_r, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, out));
  if (!weight_scales_ok(p, w_gate_scale, w_up_scale, w_down_scale)) return MOE_ERR_INVALID_ARG;
  return do_layer(p, x, x_scale, w_r, bias, w_gate, w_up, w_down, w_gate_scale, w_up_scale, w_down_scale,
                  ws_gate, ws_up, ws_down, out, topk_ids_out,
                  topk_w_out, counts_out, ws, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_layer_forward_host(const moe_params_t* p, const void* x_host, const float* x_scale_host,
                                    const void* w_r, const float* bias, const void* w_gate, const void* w_up,
                                    const void* w_down, const void* w_gate_scale, const void* w_up_scale,
                                    const void* w_down_scale, const void* ws_gate, const void* ws_up,
                                    const void* ws_down, void* out_host, void* ws, size_t ws_bytes,
                                    void* stream) {
  MOE_TRY(validate(p));
  MOE_TRY(check_ws(p, ws, ws_bytes, true));
  if (p->T == 0) return MOE_OK;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  if (is_fp8(p) && !x_scale_host) return MOE_ERR_INVALID_ARG;
  if (!weight_scales_ok(p, w_gate_scale, w_up_scale, w_down_scale)) return MOE_ERR_INVALID_ARG;
  const Layout L = layout(p);
  void* x_dev = at<void>(ws, L.x_stage[0]);
  float* xs_dev = is_fp8(p) ? at<float>(ws, L.x_scale_stage[0]) : nullptr;
  void* out_dev = at<void>(ws, L.out_stage[0]);
  MOE_TRY(check_layer_args(p, x_dev, xs_dev, w_r, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, out_dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t xbytes = static_cast<size_t>(p->T) * p->H * (is_fp8(p) ? 1 : 2);
  MOE_CUDA(cudaMemcpyAsync(x_dev, x_host, xbytes, cudaMemcpyHostToDevice, st));
  if (is_fp8(p))
    MOE_CUDA(cudaMemcpyAsync(xs_dev, x_scale_host, static_cast<size_t>(p->T) * (p->H / 128) * sizeof(float),
                             cudaMemcpyHostToDevice, st));
  MOE_TRY(do_layer(p, x_dev, xs_dev, w_r, bias, w_gate, w_up, w_down, w_gate_scale, w_up_scale, w_down_scale,
                   ws_gate, ws_up, ws_down, out_dev, nullptr, nullptr, nullptr, ws, st));
  MOE_CUDA(cudaMemcpyAsync(out_host, out_dev, static_cast<size_t>(p->T) * p->H * 2, cudaMemcpyDeviceToHost, st));
  return MOE_OK;
}

moe_status_t moe_layer_forward_host_batches(const moe_params_t* p, int32_t n_batches, const void* const* x_host,
                                            const float* const* x_scale_host, const void* w_r, const float* bias,
                                            const void* w_gate, const void* w_up, const void* w_down,
                                            const void* w_gate_scale, const void* w_up_scale,
                                            const void* w_down_scale, const void* ws_gate, const void* ws_up,
                                            const void* ws_down, void* const* out_host, void* ws, size_t ws_bytes,
                                            void* stream) {
  MOE_TRY(validate(p));
  MOE_TRY(check_ws(p, ws, ws_bytes, true));
  if (n_batches < 0) return MOE_ERR_INVALID_ARG;
  if (n_batches == 0 || p->T == 0) return MOE_OK;
  if (!x_host || !out_host || (is_fp8(p) && !x_scale_host)) return MOE_ERR_INVALID_ARG;
  for (int32_t b = 0; b < n_batches; ++b)
    if (!x_host[b] || !out_host[b] || (is_fp8(p) && !x_scale_host[b])) return MOE_ERR_INVALID_ARG;
  if (!weight_scales_ok(p, w_gate_scale, w_up_scale, w_down_scale)) return MOE_ERR_INVALID_ARG;
  const Layout L = layout(p);
  for (int slot = 0; slot < 2; ++slot)
    MOE_TRY(check_layer_args(p, at<void>(ws, L.x_stage[slot]),
                             is_fp8(p) ? at<float>(ws, L.x_scale_stage[slot]) : nullptr, w_r, w_gate, w_up, w_down,
                             ws_gate, ws_up, ws_down, at<void>(ws, L.out_stage[slot])));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_copy_mu);
  const Copies* c = copies_for_current_device();
  if (c == nullptr) return MOE_ERR_CUDA;
  const size_t xbytes = static_cast<size_t>(p->T) * p->H * (is_fp8(p) ? 1 : 2);
  const size_t sbytes = static_cast<size_t>(p->T) * (p->H / 128) * sizeof(float);
  const size_t obytes = static_cast<size_t>(p->T) * p->H * 2;
  // the first copy in comes after the work already on the caller's stream
  MOE_CUDA(cudaEventRecord(c->fork, st));
  MOE_CUDA(cudaStreamWaitEvent(c->in, c->fork, 0));
  MOE_CUDA(cudaStreamWaitEvent(c->out, c->fork, 0));
  moe_status_t status = MOE_OK;
  for (int32_t b = 0; b < n_batches && status == MOE_OK; ++b) {
    const int slot = b & 1;
    void* x_dev = at<void>(ws, L.x_stage[slot]);
    float* xs_dev = is_fp8(p) ? at<float>(ws, L.x_scale_stage[slot]) : nullptr;
    void* out_dev = at<void>(ws, L.out_stage[slot]);
    // in: the slot's activations were read by the layer of batch b-2 (done[slot])
    if (b >= 2) MOE_CUDA(cudaStreamWaitEvent(c->in, c->done[slot], 0));
    MOE_CUDA(cudaMemcpyAsync(x_dev, x_host[b], xbytes, cudaMemcpyHostToDevice, c->in));
    if (is_fp8(p)) MOE_CUDA(cudaMemcpyAsync(xs_dev, x_scale_host[b], sbytes, cudaMemcpyHostToDevice, c->in));
    MOE_CUDA(cudaEventRecord(c->landed[slot], c->in));
    // the layer: after its activations landed and the slot's previous output left
    MOE_CUDA(cudaStreamWaitEvent(st, c->landed[slot], 0));
    if (b >= 2) MOE_CUDA(cudaStreamWaitEvent(st, c->left[slot], 0));
    status = do_layer(p, x_dev, xs_dev, w_r, bias, w_gate, w_up, w_down, w_gate_scale, w_up_scale, w_down_scale,
                      ws_gate, ws_up, ws_down, out_dev, nullptr, nullptr, nullptr, ws, st);
    MOE_CUDA(cudaEventRecord(c->done[slot], st));
    // out
    MOE_CUDA(cudaStreamWaitEvent(c->out, c->done[slot], 0));
    MOE_CUDA(cudaMemcpyAsync(out_host[b], out_dev, obytes, cudaMemcpyDeviceToHost, c->out));
    MOE_CUDA(cudaEventRecord(c->left[slot], c->out));
  }
  // the caller's stream passes the call once every output has left
  MOE_CUDA(cudaStreamWaitEvent(st, c->left[0], 0));
  if (n_batches > 1) MOE_CUDA(cudaStreamWaitEvent(st, c->left[1], 0));
  return status;
}

moe_status_t moe_get_device_status(const void* ws, void* stream, int32_t* host_status) {
  if (!ws || !host_status) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  MOE_CUDA(cudaMemcpy(host_status, ws, sizeof(int32_t), cudaMemcpyDeviceToHost));
  return MOE_OK;
}

moe_status_t moe_clear_device_status(void* ws, void* stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)));
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
    case MOE_ERR_DEVICE: return "device detected bad input";
  }
  return "unknown status";
}

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status_t moe_selftest_bounded_wait(void* ws, int32_t limit_ms, void* stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0 || limit_ms < 1 || limit_ms > 2000)
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_bounded_wait_selftest(static_cast<int32_t*>(ws), 1000000LL * limit_ms,
                                                  static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_prepare_fp4_scales(const void* scale_words, int64_t rows, int32_t K, void* atoms, void* stream) {
  if (!scale_words || !atoms || rows <= 0 || rows % 128 != 0 || K <= 0 || K % 128 != 0) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scale_words) & 3u) != 0 || !aligned16(atoms)) return MOE_ERR_INVALID_ARG;
  if (rows > (1LL << 40) / K) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_fp4_scale_atoms(static_cast<const uint32_t*>(scale_words), rows, K,
                                            static_cast<uint8_t*>(atoms), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_trace_enable(uint32_t kernel_mask, int32_t capacity) {
  if (capacity <= 0 || capacity > (1 << 20)) return MOE_ERR_INVALID_ARG;
  Trace& t = g_trace;
  if (static_cast<int>(t.kid.size()) < capacity) {
    const size_t have = t.ev.size();
    t.ev.resize(2 * static_cast<size_t>(capacity));
    for (size_t i = have; i < t.ev.size(); ++i)
      if (cudaEventCreate(&t.ev[i]) != cudaSuccess) return MOE_ERR_CUDA;
    t.kid.resize(capacity);
  }
  t.cap = capacity;
  t.mask = kernel_mask;
  t.n = 0;
  t.on = true;
  return MOE_OK;
}

moe_status_t moe_trace_disable(void) {
  g_trace.on = false;
  return MOE_OK;
}

int32_t moe_trace_collect(int32_t* kernel_ids, float* ms, int32_t max_out) {
  Trace& t = g_trace;
  int32_t n = 0;
  for (int i = 0; i < t.n && n < max_out; ++i) {
    if (cudaEventSynchronize(t.ev[2 * i + 1]) != cudaSuccess) break;
    float v = 0.f;
    if (cudaEventElapsedTime(&v, t.ev[2 * i], t.ev[2 * i + 1]) != cudaSuccess) break;
    if (kernel_ids) kernel_ids[n] = t.kid[i];
    if (ms) ms[n] = v;
    ++n;
  }
  t.n = 0;
  return n;
}

int32_t moe_layer_launch_count(const moe_params_t* p) {
  if (validate(p) != MOE_OK) return -1;
  if (p->T == 0) return 0;
  int n = 2;                                 // router GEMM, top-k
  if (is_fp8(p)) n += is_fp4(p) ? 1 : 4;     // dequantise x for the router (and the scale atoms
                                             // of the three e4m3 weights; x's come with the copy)
  const long long P = static_cast<long long>(p->T) * p->K;
  n += P <= kSmallPairs ? 2 : 4;             // count, scan, rank (one kernel for few pairs), gather
  n += 2;                                    // gate/up, down
  if (p->I_shared > 0 && !shared_merged(p)) n += 2;  // shared gate/up, down (unless in the routed ones)
  n += 1;                                    // combine
  if (p->masked_cap > 0) n += 1;             // compact GEMM schedule of the masked layout
  return n;
}

}  // extern "C"
