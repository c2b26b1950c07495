// C ABI of the fused chunked KL loss: argument checks, workspace layout,
// work planner, TMA descriptors and the token-chunk scheduler of the backward.
//
// The forward needs no token chunking: its per-row state (running max,
// sum-exp, gathered logit) is O(N), and the vocabulary is swept tile by tile
// with an online log-sum-exp (the vocabulary-axis chunking of the llm-wiki
// note, section "Fused Chunked KL").  The backward loops over token chunks
// (the sequence-axis chunking of the mind-verse.de article, three-variant list,
// "Fused chunked KL"): each chunk's logits are recomputed, turned into the
// gradient G on chip, written once as bf16 into an N-independent chunk buffer,
// and consumed by the dHidden and dW GEMMs before the next chunk overwrites it.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/kdkl.h"
#include "kdkl_internal.h"

namespace kdkl {
namespace {

thread_local char g_last_error[256] = {0};

kdkl_status fail(kdkl_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

kdkl_status ok() {
  g_last_error[0] = 0;
  return KDKL_OK;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int64_t kDefaultChunk = 8192;
constexpr int kDefaultSyncWindow = 1;      // row-stream GEMMs: tiles (measured best of 0, 1, 2, 4, 8)
constexpr int kDefaultSyncKWindow = 64;    // tile-mode GEMMs: reduction blocks (measured best of 0, 8 ... 256)
constexpr int kSplitGroupMB = 32;          // split-major GEMMs: hidden rows per row-block group
constexpr int kTileColGroup = 0;           // dHidden / dW: column tiles per group (0 = all)
constexpr int kDieOrder = 0;               // GEMM groups numbered by block index
constexpr int64_t kMaxRows = (int64_t(1) << 31) - 256;
constexpr int32_t kMaxV = (int32_t(1) << 30);

// --------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 map: `inner` contiguous elements per row, `outer` rows, row pitch in elements.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_elems,
              uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_elems * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same for an fp32 matrix.
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_elems,
              uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_elems * 4};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// --------------------------------------------------------------- planner
struct Device {
  int id = 0;
  int sms = 0;
  int cc_major = 0;
};

kdkl_status current_device(Device& dv) {
  if (cudaGetDevice(&dv.id) != cudaSuccess) return fail(KDKL_ERR_UNSUPPORTED, "no CUDA device is current");
  if (cudaDeviceGetAttribute(&dv.sms, cudaDevAttrMultiProcessorCount, dv.id) != cudaSuccess ||
      cudaDeviceGetAttribute(&dv.cc_major, cudaDevAttrComputeCapabilityMajor, dv.id) != cudaSuccess)
    return fail(KDKL_ERR_CUDA, "cudaDeviceGetAttribute failed");
  if (dv.cc_major != 10) return fail(KDKL_ERR_UNSUPPORTED, "kdkl needs an sm_100 device (found cc %d.x)", dv.cc_major);
  return KDKL_OK;
}

// A tuning knob: the environment variable `name` as a non-negative integer, or dflt.
int env_window(const char* name, int dflt) {
  const char* e = std::getenv(name);
  int v = dflt;
  if (e && *e) v = std::atoi(e);
  return v < 0 ? 0 : v;
}

// Vocabulary splits for a row-stream kernel over `rb` row blocks and `vt`
// vocabulary tiles: balance the per-group tile count over `ctas` CTA groups
// (single CTAs or CTA pairs), and keep at least enough splits that the hidden
// rows in flight stay small next to L2.  `units_cap` bounds rb * splits.
int pick_splits(int64_t rb, int vt, int ctas, int d, int64_t units_cap, int rows_per_block, int s_floor = 1) {
  // Fewer splits mean fewer passes over W, hence less DRAM traffic and power,
  // but more hidden rows in flight.  Measured on B200 (forward, steady state):
  // the fastest split counts were 2 at (N, d, V) = (131072, 2880, 201088),
  // 3 at (131072, 4096, 128256) and 4 at (32768, 4096, 128256), i.e. 37-55 MB of
  // hidden rows in flight, 3-9 % faster than at 18-20 MB.  KDKL_ROWS_BUDGET_MB
  // overrides the budget, for tuning.
  const double rows_bytes = static_cast<double>(rows_per_block) * d * 2.0;
  static const int budget_mb = env_window("KDKL_ROWS_BUDGET_MB", 55);   // override for tuning
  const double budget = budget_mb * 1024.0 * 1024.0;
  int s_min = static_cast<int>(std::ceil(ctas * rows_bytes / budget));
  if (s_min < s_floor) s_min = s_floor;
  if (s_min < 1) s_min = 1;
  int s_max = static_cast<int>(units_cap / rb);
  if (s_max > vt) s_max = vt;
  if (s_max < 1) s_max = 1;
  if (s_min > s_max) s_min = s_max;
  // Tile-count cost of the slowest group; more splits also mean fewer groups
  // sharing each W tile (more W traffic), so take the fewest splits whose cost
  // is within 1 % of the best.
  auto cost = [&](int s) {
    const int64_t units = rb * s;
    const int64_t waves = (units + ctas - 1) / ctas;
    const int64_t per_unit = (vt + s - 1) / s;
    return static_cast<double>(waves * per_unit);
  };
  double best_cost = 1e300;
  for (int s = s_min; s <= s_max; ++s) best_cost = std::min(best_cost, cost(s));
  for (int s = s_min; s <= s_max; ++s)
    if (cost(s) <= best_cost * 1.01) return s;
  return s_min;
}

// Tile widths (N, over d) of the dHidden / dW GEMMs.  CTA pairs (cta_group::2,
// 256-row tiles) run any width in kPairTileN; single CTAs, used only on a
// device with one SM, run 256, 192 or 128.
constexpr int kPairTileN[] = {256, 240, 224, 192, 160, 128};

bool pair_tile_n_ok(int bn) {
  for (int t : kPairTileN)
    if (t == bn) return true;
  return false;
}

int pick_bn_single(int d) {
  const int64_t pad256 = static_cast<int64_t>((d + 255) / 256) * 256;
  const int64_t pad192 = static_cast<int64_t>((d + 191) / 192) * 192;
  const int64_t pad128 = static_cast<int64_t>((d + 127) / 128) * 128;
  const int64_t best_narrow = pad192 < pad128 ? pad192 : pad128;
  if (pad256 * 8 <= best_narrow * 9) return 256;
  return pad192 <= pad128 ? 192 : 128;
}

// Whether a GEMM runs as CTA pairs (256-row tiles, cta_group::2) or single
// CTAs (128-row tiles).
struct Pairing {
  bool pair;
  int rows;     // rows of one tile / unit
  int groups;   // CTA groups that run at once (pairs or single CTAs)
  int b_rows;   // rows of the K-major B box one CTA loads
  int grid(int64_t units) const {
    const int64_t g = units < groups ? units : groups;
    return static_cast<int>(pair ? 2 * g : g);
  }
};

Pairing pairing(int sms, int bn) {
  Pairing p;
  p.pair = sms >= 2;
  p.rows = p.pair ? 2 * kBM : kBM;
  p.groups = p.pair ? sms / 2 : sms;
  p.b_rows = p.pair ? bn / 2 : bn;
  return p;
}

// Backward plan: tile width of the dHidden / dW GEMMs and tokens per chunk.
//
// Cost model (seconds, at an assumed kPlanSmRate flop/s per SM): per chunk of
// nc tokens, the dHidden GEMM runs ceil(ceil(nc / rows) * nt / groups) waves of
// tiles that each reduce over the whole vocabulary (2 * rows * bn * V flops),
// and the dW GEMM ceil(ceil(V / rows) * nt / groups) waves of tiles reducing
// over the chunk (2 * rows * bn * nc flops); a tile of width bn runs at
// tile_efficiency(bn) of the 256-wide tile's flop rate, every tile adds
// kPlanTileFixed and every chunk kPlanChunkFixed.  With V in the hundreds of
// thousands a dHidden tile runs for about a millisecond, so a partly filled
// last wave costs more than an extra chunk.  Among plans within 1 % of the
// cheapest, the widest tile and then the largest chunk win.
constexpr double kPlanSmRate = 8.0e12;
constexpr double kPlanTileFixed = 2.0e-6;
constexpr double kPlanChunkFixed = 40.0e-6;

// Flop rate of a CTA-pair tile of width bn relative to the 256-wide tile, as
// measured on B200 from the dHidden and dW kernels' times at equal work, scaled
// by the sampled SM clock (d = 2880, 3584 and 4096): narrower tiles stream the
// same A operand for fewer MMA flops and turn their pipeline stages over faster.
double tile_efficiency(int bn) {
  switch (bn) {
    case 256: return 1.0;
    case 240: return 0.87;
    case 224: return 0.92;
    case 192: return 0.75;
    case 160: return 0.67;
    default: return 0.5;
  }
}

double backward_cost(int64_t N, int d, int V, int bn, int64_t chunk, const Pairing& p) {
  const double rate = kPlanSmRate * (p.pair ? 2.0 : 1.0) * tile_efficiency(bn);
  const int64_t nt = (d + bn - 1) / bn;
  const int64_t vb = (V + p.rows - 1) / p.rows;
  auto chunk_cost = [&](int64_t nc) {
    const int64_t rb = (nc + p.rows - 1) / p.rows;
    const int64_t w_dh = (rb * nt + p.groups - 1) / p.groups;
    const int64_t w_dw = (vb * nt + p.groups - 1) / p.groups;
    const double t_dh = 2.0 * p.rows * bn * static_cast<double>(V) / rate + kPlanTileFixed;
    const double t_dw = 2.0 * p.rows * bn * static_cast<double>(nc) / rate + kPlanTileFixed;
    return static_cast<double>(w_dh) * t_dh + static_cast<double>(w_dw) * t_dw + kPlanChunkFixed;
  };
  const int64_t full = N / chunk, rest = N % chunk;
  return static_cast<double>(full) * chunk_cost(chunk) + (rest ? chunk_cost(rest) : 0.0);
}

struct BackwardPlan {
  int bn;
  int64_t chunk;
};

// `cap` = the workspace's chunk capacity (L.chunk); `auto_chunk` = chunk_tokens was 0.
BackwardPlan plan_backward(int64_t N, int d, int V, int64_t cap, bool auto_chunk, int forced_bn, int sms) {
  BackwardPlan best{256, cap};
  if (sms < 2) {
    best.bn = pick_bn_single(d);
    return best;
  }
  const Pairing p = pairing(sms, 256);
  struct Cand {
    double cost;
    int bn;
    int64_t chunk;
  };
  Cand cands[6 * 64];
  int n = 0;
  double lo = 1e300;
  for (int bn : kPairTileN) {
    if (forced_bn && bn != forced_bn) continue;
    // chunk candidates: the capacity itself, then multiples of the tile height below it
    int64_t ch = cap;
    int taken = 0;
    while (ch >= 1 && taken < 64) {
      const double cost = backward_cost(N, d, V, bn, ch, p);
      cands[n++] = Cand{cost, bn, ch};
      lo = cost < lo ? cost : lo;
      ++taken;
      if (!auto_chunk) break;
      const int64_t next = (ch - 1) / p.rows * p.rows;
      if (next < p.rows) break;
      ch = next;
    }
  }
  bool have = false;
  for (int i = 0; i < n; ++i) {
    if (cands[i].cost > lo * 1.01) continue;
    if (!have || cands[i].bn > best.bn || (cands[i].bn == best.bn && cands[i].chunk > best.chunk)) {
      best.bn = cands[i].bn;
      best.chunk = cands[i].chunk;
      have = true;
    }
  }
  return best;
}

kdkl_status check_shapes(int64_t N, int32_t d, int32_t V, int32_t K, float tau) {
  if (N < 0 || N > kMaxRows) return fail(KDKL_ERR_SHAPE, "N=%lld outside [0, %lld]", (long long)N, (long long)kMaxRows);
  if (d < 8 || d % 8 != 0) return fail(KDKL_ERR_SHAPE, "d=%d must be a positive multiple of 8", d);
  if (V < 1 || V > kMaxV) return fail(KDKL_ERR_SHAPE, "V=%d outside [1, 2^30]", V);
  if (K < 1 || K > kMaxK) return fail(KDKL_ERR_SHAPE, "K=%d outside [1, %d]", K, kMaxK);
  if (K > V) return fail(KDKL_ERR_SHAPE, "K=%d larger than V=%d", K, V);
  if (!std::isfinite(tau) || !(tau > 0.f)) return fail(KDKL_ERR_SHAPE, "tau must be finite and > 0");
  return KDKL_OK;
}

struct Common {
  const void* hidden;
  const void* W;
  const void* idx;
  const void* logit;
  const uint8_t* mask;
  int64_t N;
  int32_t d, V, K;
  float tau;
  void* ws;
  size_t ws_bytes;
  kdkl_options opt;
};

kdkl_options default_options() {
  kdkl_options o;
  std::memset(&o, 0, sizeof(o));
  o.cache_format = KDKL_CACHE_I32_F32;
  o.student_tau = 1.0f;
  o.kd_weight = 1.0f;
  o.kd_scale_tau_sq = 0;
  o.ce_weight = 0.0f;
  o.labels = nullptr;
  o.n_valid_global = nullptr;
  o.bwd_tile_n = 0;
  return o;
}

float kd_gamma(const kdkl_options& o) {
  return o.kd_weight * (o.kd_scale_tau_sq ? o.student_tau * o.student_tau : 1.0f);
}

kdkl_status check_options(const Common& c) {
  const kdkl_options& o = c.opt;
  if (o.cache_format != KDKL_CACHE_I32_F32 && o.cache_format != KDKL_CACHE_U16_BF16)
    return fail(KDKL_ERR_UNSUPPORTED, "unknown cache_format %d", o.cache_format);
  if (o.cache_format == KDKL_CACHE_U16_BF16 && c.V > 65536)
    return fail(KDKL_ERR_SHAPE, "the 16-bit index cache needs V <= 65536 (V=%d)", c.V);
  if (!std::isfinite(o.student_tau) || !(o.student_tau > 0.f))
    return fail(KDKL_ERR_SHAPE, "student_tau must be finite and > 0");
  if (!std::isfinite(o.kd_weight) || o.kd_weight < 0.f || !std::isfinite(o.ce_weight) || o.ce_weight < 0.f)
    return fail(KDKL_ERR_SHAPE, "kd_weight and ce_weight must be finite and >= 0");
  if (o.ce_weight > 0.f && !o.labels) return fail(KDKL_ERR_NULL, "ce_weight > 0 needs labels");
  if (o.labels && !aligned(o.labels, 4)) return fail(KDKL_ERR_ALIGN, "labels must be 4-byte aligned");
  if (o.n_valid_global && !aligned(o.n_valid_global, 4)) return fail(KDKL_ERR_ALIGN, "n_valid_global must be 4-byte aligned");
  if (o.bwd_tile_n != 0 && !pair_tile_n_ok(o.bwd_tile_n))
    return fail(KDKL_ERR_UNSUPPORTED, "bwd_tile_n=%d is not 0 or one of 128, 160, 192, 224, 240, 256", o.bwd_tile_n);
  return KDKL_OK;
}

// The forward only uses the workspace before the chunk buffer, so any
// chunk_tokens value gives it enough room; the backward needs all of it.
kdkl_status check_common(const Common& c, int64_t chunk_tokens, bool need_chunk_buffer, WsLayout& L) {
  kdkl_status st = check_shapes(c.N, c.d, c.V, c.K, c.tau);
  if (st != KDKL_OK) return st;
  if (!c.hidden || !c.W || !c.idx || !c.logit || !c.mask || !c.ws)
    return fail(KDKL_ERR_NULL, "hidden, W, topk_idx, topk_logit, mask and workspace must be non-NULL");
  if (!aligned(c.hidden, 16) || !aligned(c.W, 16)) return fail(KDKL_ERR_ALIGN, "hidden and W must be 16-byte aligned");
  st = check_options(c);
  if (st != KDKL_OK) return st;
  const size_t cache_align = c.opt.cache_format == KDKL_CACHE_U16_BF16 ? 2 : 4;
  if (!aligned(c.idx, cache_align) || !aligned(c.logit, cache_align))
    return fail(KDKL_ERR_ALIGN, "topk_idx and topk_logit must be %zu-byte aligned", cache_align);
  if (!aligned(c.ws, 256)) return fail(KDKL_ERR_ALIGN, "workspace must be 256-byte aligned");
  if (chunk_tokens < 0) return fail(KDKL_ERR_SHAPE, "chunk_tokens must be >= 0");
  L = make_layout(c.N, c.d, c.V, c.K, chunk_tokens);
  const size_t need = need_chunk_buffer ? L.total : L.gbuf;
  if (c.ws_bytes < need) return fail(KDKL_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", c.ws_bytes, need);
  return KDKL_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

kdkl_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KDKL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------- timing
enum TimedKind {
  kTPrepass = 0, kTFwd, kTMerge, kTGrad, kTDh, kTDw, kTTopK, kTTopKMerge, kTFusedFwd, kTGPass, kTKinds
};
const char* const kTimedNames[kTKinds] = {"prepass",          "fwd_lse_gemm", "merge",         "bwd_grad_gemm",
                                          "bwd_dhidden_gemm", "bwd_dw_gemm",  "teacher_topk_gemm",
                                          "teacher_topk_merge", "fused_fwd_gemm", "fused_g_pass"};
struct TimingRec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<TimingRec> g_pending;
uint64_t g_launches[kTKinds] = {0};
double g_ms[kTKinds] = {0};

template <class F>
cudaError_t timed(int kind, cudaStream_t s, F&& launch) {
  bool on;
  {
    std::lock_guard<std::mutex> lk(g_tmu);
    on = g_timing;
  }
  if (!on) return launch();
  cudaEvent_t a = nullptr, b = nullptr;
  if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return cudaGetLastError();
  cudaEventRecord(a, s);
  const cudaError_t e = launch();
  cudaEventRecord(b, s);
  std::lock_guard<std::mutex> lk(g_tmu);
  g_pending.push_back({kind, a, b});
  return e;
}

// Prepass shared by forward and backward (the backward keeps no state from the forward).
kdkl_status run_prepass(const Common& c, const WsLayout& L, cudaStream_t s) {
  uint32_t* header = at<uint32_t>(c.ws, L.header);
  cudaError_t e = cudaMemsetAsync(header, 0, 256, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  e = timed(kTPrepass, s, [&] {
    return launch_prepass(c.opt.cache_format, c.idx, c.logit, c.mask, c.opt.labels, c.N, c.V, c.K, c.tau,
                          kd_gamma(c.opt), c.opt.ce_weight, at<int>(c.ws, L.sidx), at<float>(c.ws, L.sprob),
                          at<float>(c.ws, L.negent), at<float>(c.ws, L.wsum), at<uint8_t>(c.ws, L.rowmask), L.Kp,
                          header, s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "prepass launch");
  return KDKL_OK;
}

EpiParams base_params(const Common& c, const WsLayout& L) {
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.sidx = at<int>(c.ws, L.sidx);
  ep.sprob = at<float>(c.ws, L.sprob);
  ep.Kp = L.Kp;
  ep.rowmask = at<uint8_t>(c.ws, L.rowmask);
  ep.n_valid = c.opt.n_valid_global ? c.opt.n_valid_global : at<uint32_t>(c.ws, L.header) + 1;
  ep.flags = at<uint32_t>(c.ws, L.header);
  ep.inv_tau_s = 1.0f / c.opt.student_tau;
  ep.exp_scale = 1.4426950408889634f / c.opt.student_tau;
  ep.wsum = at<float>(c.ws, L.wsum);
  return ep;
}

// How far a group may run ahead of the slowest group sharing its operands (the
// lockstep; 0 = off): in tiles for the row-stream GEMMs, in 64-wide reduction blocks
// for the tile-mode ones.  KDKL_SYNC_WINDOW / KDKL_SYNC_KWINDOW override the defaults,
// for tuning.
int sync_window() {
  static int w = env_window("KDKL_SYNC_WINDOW", kDefaultSyncWindow);
  return w;
}
int sync_kwindow() {
  static int w = env_window("KDKL_SYNC_KWINDOW", kDefaultSyncKWindow);
  return w;
}

// Row blocks per group of a split-major launch: about kSplitGroupBytes of hidden rows
// (KDKL_SPLIT_GROUP_MB overrides it for tuning; 0 = one group of every row block).
// Every group streams all of W once, so smaller groups trade W passes for fewer hidden
// rows that must stay in L2 while each W tile is shared.
// Group numbering by the half of the SM ids a CTA group runs on (KDKL_DIE_ORDER, for
// tuning; 0 = by block index).
int die_order() {
  static int v = env_window("KDKL_DIE_ORDER", kDieOrder);
  return v;
}

// Column tiles per group of the dHidden / dW launches (KDKL_TILE_COL_GROUP, for tuning;
// 0 = all tiles of a row block in a row).
int tile_col_group() {
  static int g = env_window("KDKL_TILE_COL_GROUP", kTileColGroup);
  return g;
}

int split_rb_group(int d, int rows_per_block) {
  static int mb = env_window("KDKL_SPLIT_GROUP_MB", kSplitGroupMB);
  if (mb <= 0) return 0;
  const double rows_bytes = static_cast<double>(rows_per_block) * d * 2.0;
  const int g = static_cast<int>(mb * 1048576.0 / rows_bytes);
  return g < 1 ? 1 : g;
}

// L2 eviction priorities of the operand loads (KDKL_L2_HINTS, a bit mask, for tuning;
// default 0 = every load at normal priority):
//   bit 0: the hidden rows of the row-stream GEMMs (each row block is re-read for every
//          vocabulary tile of its unit) are kept with evict_last;
//   bit 1: the dW GEMM's hidden chunk (re-read by every vocabulary row block) likewise.
int l2_hint_mask() {
  static int m = [] {
    const char* e = std::getenv("KDKL_L2_HINTS");
    return (e && *e) ? std::atoi(e) : 0;
  }();
  return m;
}

// Arms the lockstep of a launch of `grid` CTAs: clears the groups' position words on
// the stream, ahead of the launch.
cudaError_t arm_sync(Sched& sc, unsigned long long* prog, int grid, bool pair, cudaStream_t s) {
  const int groups = pair ? grid / 2 : grid;
  sc.sync_window = 0;
  sc.die_order = 0;
  sc.prog = prog;
  if (sc.row_stream && (l2_hint_mask() & 1)) sc.l2_a = kL2Last;
  if (groups < 2 || groups + 2 > kSyncSlots) return cudaSuccess;
  const int w = sc.row_stream ? sync_window() : sync_kwindow();
  sc.sync_window = w > 0 ? w : 0;
  sc.die_order = die_order();
  if (sc.sync_window == 0 && sc.die_order == 0) return cudaSuccess;
  // the groups' position words and, after them, the two ticket counters of die_order
  return cudaMemsetAsync(prog, 0, static_cast<size_t>(groups + 2) * 8, s);
}

}  // namespace

WsLayout make_layout(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens) {
  (void)d;
  WsLayout L;
  L.Kp = list_pitch(K);
  const int64_t rb = (N + kBM - 1) / kBM;
  L.units_cap = rb * 8 + 4096;
  int64_t chunk = chunk_tokens > 0 ? chunk_tokens : kDefaultChunk;
  chunk = (chunk + kBM - 1) / kBM * kBM;
  const int64_t n_up = (N + kBM - 1) / kBM * kBM;
  if (chunk > n_up) chunk = n_up;
  if (chunk < kBM) chunk = kBM;
  L.chunk = chunk;
  L.Vp = (static_cast<int64_t>(V) + 63) / 64 * 64;
  size_t off = 0;
  L.header = off;
  off += 256;
  L.sync = off;
  off += static_cast<size_t>(kSyncSlots) * 8;
  L.sidx = off;
  off = align_up(off + static_cast<size_t>(N) * L.Kp * 4, 256);
  L.sprob = off;
  off = align_up(off + static_cast<size_t>(N) * L.Kp * 4, 256);
  L.negent = off;
  off = align_up(off + static_cast<size_t>(N) * 4, 256);
  L.wsum = off;
  off = align_up(off + static_cast<size_t>(N) * 4, 256);
  L.rowmask = off;
  off = align_up(off + static_cast<size_t>(N), 256);
  L.partial = off;
  off = align_up(off + static_cast<size_t>(L.units_cap) * kBM * 3 * 4, 256);
  L.blocksum = off;
  off = align_up(off + static_cast<size_t>((N + 255) / 256 + 1) * 8, 256);
  L.gbuf = off;
  off = align_up(off + static_cast<size_t>(L.chunk) * L.Vp * 2, 256);
  L.total = off;
  return L;
}

void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

}  // namespace kdkl

using namespace kdkl;

extern "C" {

size_t kdkl_workspace_bytes(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens) {
  if (check_shapes(N, d, V, K, 1.0f) != KDKL_OK || chunk_tokens < 0) return 0;
  return make_layout(N, d, V, K, chunk_tokens).total;
}

const char* kdkl_status_string(kdkl_status s) {
  switch (s) {
    case KDKL_OK: return "KDKL_OK";
    case KDKL_ERR_NULL: return "KDKL_ERR_NULL";
    case KDKL_ERR_SHAPE: return "KDKL_ERR_SHAPE";
    case KDKL_ERR_ALIGN: return "KDKL_ERR_ALIGN";
    case KDKL_ERR_UNSUPPORTED: return "KDKL_ERR_UNSUPPORTED";
    case KDKL_ERR_WORKSPACE: return "KDKL_ERR_WORKSPACE";
    case KDKL_ERR_CUDA: return "KDKL_ERR_CUDA";
  }
  return "KDKL_ERR_UNKNOWN";
}

const char* kdkl_last_error(void) { return g_last_error; }

static kdkl_status forward_impl(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                                const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                                const kdkl_options* options, float* loss, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream) {
  const Common c{hidden,    W,         topk_idx,        topk_logit, mask, N, d, V, K, tau,
                 workspace, workspace_bytes, options ? *options : default_options()};
  WsLayout L;
  kdkl_status st = check_common(c, 0, false, L);
  if (st != KDKL_OK) return st;
  if (!loss || !lse) return fail(KDKL_ERR_NULL, "loss and lse must be non-NULL");
  if (!aligned(loss, 4) || !aligned(lse, 4)) return fail(KDKL_ERR_ALIGN, "loss and lse must be 4-byte aligned");
  Device dv;
  if ((st = current_device(dv)) != KDKL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (N == 0) {
    if ((e = cudaMemsetAsync(workspace, 0, 256, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    if ((e = cudaMemsetAsync(loss, 0, sizeof(float), s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    return ok();
  }
  if ((st = run_prepass(c, L, s)) != KDKL_OK) return st;

  const Pairing pr = pairing(dv.sms, 256);
  const int64_t rb = (N + pr.rows - 1) / pr.rows;
  const int vt = (V + 255) / 256;
  const int splits = pick_splits(rb, vt, pr.groups, d, L.units_cap * kBM / pr.rows, pr.rows);
  Sched sc;
  sc.units = static_cast<int>(rb * splits);
  sc.splits = splits;
  sc.n_tiles = vt;
  sc.k_blocks = (d + kBK - 1) / kBK;
  sc.row_stream = kRowMajor;
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, hidden, d, N, d, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tmB, W, d, V, d, kBK, pr.b_rows, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(KDKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (hidden/W)");
  EpiParams ep = base_params(c, L);
  ep.M = static_cast<int>(N);
  ep.Ncols = V;
  ep.row_offset = 0;
  float* part = at<float>(workspace, L.partial);
  const size_t plane = static_cast<size_t>(L.units_cap) * kBM;
  ep.part_m = part;
  ep.part_s = part + plane;
  ep.part_a = part + 2 * plane;
  ep.part_cap = static_cast<int64_t>(plane);
  const int grid = pr.grid(sc.units);
  if ((e = arm_sync(sc, at<unsigned long long>(workspace, L.sync), grid, pr.pair, s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync");
  if ((e = timed(kTFwd, s, [&] { return launch_gemm(kEpiLse, 256, pr.pair, tmA, tmB, tmA, sc, ep, grid, s); })) !=
      cudaSuccess)
    return cuda_fail(e, "forward GEMM launch");
  uint32_t* header = at<uint32_t>(workspace, L.header);
  if ((e = timed(kTMerge, s, [&] {
         return launch_merge(ep.part_m, ep.part_s, ep.part_a, splits, pr.rows, c.opt.student_tau,
                             at<float>(workspace, L.negent), at<float>(workspace, L.wsum),
                             at<uint8_t>(workspace, L.rowmask), N, lse, loss, at<double>(workspace, L.blocksum),
                             header, ep.n_valid, 0, 0, static_cast<int64_t>(plane), s);
       })) != cudaSuccess)
    return cuda_fail(e, "merge launch");
  return ok();
}

kdkl_status kdkl_forward(const void* hidden, const void* W, const int32_t* topk_idx, const float* topk_logit,
                         const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau, float* loss,
                         float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(hidden, W, topk_idx, topk_logit, mask, N, d, V, K, tau, nullptr, loss, lse, workspace,
                      workspace_bytes, stream);
}

kdkl_status kdkl_forward_ex(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                            const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                            const kdkl_options* options, float* loss, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return forward_impl(hidden, W, topk_idx, topk_logit, mask, N, d, V, K, tau, options, loss, lse, workspace,
                      workspace_bytes, stream);
}

// The chunk's dHidden rows (= G W, bf16) and its dW term (dW (+)= G^T hidden_chunk,
// fp32 read-modify-write in chunk order; the first chunk overwrites), from the
// chunk's G in the chunk buffer.
static kdkl_status run_dh_dw(const EpiParams& ep0, const Pairing& pd, int bn, int32_t V, int32_t d, int64_t c0,
                             int64_t nc, const CUtensorMap& tmG_k, const CUtensorMap& tmG_mn,
                             const CUtensorMap& tmW_mn, const CUtensorMap& tmH_mn, void* dHidden, float* dW,
                             unsigned long long* prog, cudaStream_t s) {
  const int nt = (d + bn - 1) / bn;
  cudaError_t e;
  {
    const int64_t rbc = (nc + pd.rows - 1) / pd.rows;
    Sched sc{static_cast<int>(rbc * nt), 1, nt, static_cast<int>((V + kBK - 1) / kBK), 0};
    sc.col_group = tile_col_group();
    EpiParams ep = ep0;
    ep.M = static_cast<int>(nc);
    ep.Ncols = d;
    ep.row_offset = c0;
    ep.dH = static_cast<uint16_t*>(dHidden);
    ep.ldo = d;
    const int grid = pd.grid(sc.units);
    if ((e = arm_sync(sc, prog, grid, pd.pair, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    if ((e = timed(kTDh, s, [&] {
           return launch_gemm(kEpiStoreBf16, bn, pd.pair, tmG_k, tmW_mn, tmG_k, sc, ep, grid, s);
         })) != cudaSuccess)
      return cuda_fail(e, "dHidden GEMM launch");
  }
  {
    const int64_t vb = (V + pd.rows - 1) / pd.rows;
    Sched sc{static_cast<int>(vb * nt), 1, nt, static_cast<int>((nc + kBK - 1) / kBK), 0};
    sc.col_group = tile_col_group();
    if (l2_hint_mask() & 2) sc.l2_b = kL2Last;
    EpiParams ep = ep0;
    ep.M = V;
    ep.Ncols = d;
    ep.row_offset = 0;
    ep.dW = dW;
    ep.ldo = d;
    ep.accumulate = c0 > 0 ? 1 : 0;
    // dW blocks of 32 rows x 32 fp32 columns, 128-byte swizzle: the epilogue's TMA loads
    // of the old values and stores of the new ones
    CUtensorMap tmDW;
    if (!make_map_f32(&tmDW, dW, d, V, d, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(KDKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (dW)");
    const int grid = pd.grid(sc.units);
    if ((e = arm_sync(sc, prog, grid, pd.pair, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    if ((e = timed(kTDw, s, [&] {
           return launch_gemm(kEpiRmwF32, bn, pd.pair, tmG_mn, tmH_mn, tmDW, sc, ep, grid, s);
         })) != cudaSuccess)
      return cuda_fail(e, "dW GEMM launch");
  }
  return KDKL_OK;
}

static kdkl_status backward_impl(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                                 const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                                 const kdkl_options* options, const float* lse, const float* grad_loss,
                                 void* dHidden, float* dW, int64_t chunk_tokens, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  const Common c{hidden,    W,         topk_idx,        topk_logit, mask, N, d, V, K, tau,
                 workspace, workspace_bytes, options ? *options : default_options()};
  WsLayout L;
  kdkl_status st = check_common(c, chunk_tokens, true, L);
  if (st != KDKL_OK) return st;
  if (!lse || !dHidden || !dW) return fail(KDKL_ERR_NULL, "lse, dHidden and dW must be non-NULL");
  if (!aligned(lse, 4) || (grad_loss && !aligned(grad_loss, 4)))
    return fail(KDKL_ERR_ALIGN, "lse and grad_loss must be 4-byte aligned");
  if (!aligned(dHidden, 16) || !aligned(dW, 16)) return fail(KDKL_ERR_ALIGN, "dHidden and dW must be 16-byte aligned");
  Device dv;
  if ((st = current_device(dv)) != KDKL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (N == 0) {
    if ((e = cudaMemsetAsync(workspace, 0, 256, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    if ((e = cudaMemsetAsync(dW, 0, static_cast<size_t>(V) * d * sizeof(float), s)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    return ok();
  }
  if ((st = run_prepass(c, L, s)) != KDKL_OK) return st;

  uint16_t* gbuf = at<uint16_t>(workspace, L.gbuf);
  const Pairing pg = pairing(dv.sms, 256);          // logit recompute (always 256-wide vocabulary tiles)
  const BackwardPlan plan = plan_backward(N, d, V, L.chunk, chunk_tokens == 0, c.opt.bwd_tile_n, dv.sms);
  const int bn = plan.bn;
  const int64_t chunk = plan.chunk;
  const Pairing pd = pairing(dv.sms, bn);       // dHidden and dW GEMMs
  CUtensorMap tmW_k;  // W as K-major B of the logit recompute
  CUtensorMap tmW_mn; // W as MN-major B of dHidden = G W
  if (!make_map(&tmW_k, W, d, V, d, kBK, pg.b_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tmW_mn, W, d, V, d, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(KDKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (W)");
  const int vt = (V + 255) / 256;
  EpiParams ep0 = base_params(c, L);
  ep0.lse = lse;
  ep0.grad_loss = grad_loss;

  for (int64_t c0 = 0; c0 < N; c0 += chunk) {
    const int64_t nc = (N - c0) < chunk ? (N - c0) : chunk;
    const void* hc = static_cast<const uint8_t*>(hidden) + static_cast<size_t>(c0) * d * 2;
    CUtensorMap tmH_k, tmH_mn, tmG_store, tmG_k, tmG_mn;
    if (!make_map(&tmH_k, hc, d, nc, d, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmH_mn, hc, d, nc, d, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmG_store, gbuf, V, nc, L.Vp, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&tmG_k, gbuf, V, nc, L.Vp, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmG_mn, gbuf, V, nc, L.Vp, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(KDKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (chunk maps)");

    // (1) recompute the chunk's logits and form G (bf16) in the chunk buffer
    {
      const int64_t rbc = (nc + pg.rows - 1) / pg.rows;
      const int splits = pick_splits(rbc, vt, pg.groups, d, L.units_cap * kBM / pg.rows, pg.rows);
      // a chunk's hidden rows fit in L2, so all its row blocks sweep each split together
      Sched sc{static_cast<int>(rbc * splits), splits, vt, (d + kBK - 1) / kBK, kSplitMajor};
      sc.rb_group = split_rb_group(d, pg.rows);
      EpiParams ep = ep0;
      ep.M = static_cast<int>(nc);
      ep.Ncols = V;
      ep.row_offset = c0;
      const int grid = pg.grid(sc.units);
      if ((e = arm_sync(sc, at<unsigned long long>(workspace, L.sync), grid, pg.pair, s)) != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync");
      if ((e = timed(kTGrad, s, [&] {
             return launch_gemm(kEpiGrad, 256, pg.pair, tmH_k, tmW_k, tmG_store, sc, ep, grid, s);
           })) != cudaSuccess)
        return cuda_fail(e, "gradient GEMM launch");
    }
    // (2) dHidden rows of the chunk = G W; (3) dW (+)= G^T hidden_chunk
    if ((st = run_dh_dw(ep0, pd, bn, V, d, c0, nc, tmG_k, tmG_mn, tmW_mn, tmH_mn, dHidden, dW,
                        at<unsigned long long>(workspace, L.sync), s)) != KDKL_OK)
      return st;
  }
  return ok();
}

// ---------------------------------------------------------------- fused forward + backward
// The step without the backward's logit recompute: per token chunk, one GEMM
// computes the chunk's logits once, folds them into the online log-sum-exp and
// gather (as the forward) and stores them (fp32) in a chunk buffer; the chunk's
// merge completes its rows' lse (and the loss, after the last chunk); G is then
// formed from the stored logits and the chunk's dHidden / dW GEMMs run as in the
// backward.  The chunk buffer is N-independent, so peak memory stays linear in N.
// Fused chunks are multiples of the merge's 256-row block.
static int64_t fused_chunk_tokens(int64_t chunk_tokens) {
  return chunk_tokens > 0 ? (chunk_tokens + 255) / 256 * 256 : 0;
}

static size_t fused_logit_offset(const WsLayout& L) { return align_up(L.total, 256); }

static size_t fused_total(const WsLayout& L) {
  return fused_logit_offset(L) + static_cast<size_t>(L.chunk) * L.Vp * sizeof(float);
}

static kdkl_status forward_backward_impl(const void* hidden, const void* W, const void* topk_idx,
                                         const void* topk_logit, const uint8_t* mask, int64_t N, int32_t d,
                                         int32_t V, int32_t K, float tau, const kdkl_options* options,
                                         const float* grad_loss, float* loss, float* lse, void* dHidden, float* dW,
                                         int64_t chunk_tokens, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  const Common c{hidden,    W,         topk_idx,        topk_logit, mask, N, d, V, K, tau,
                 workspace, workspace_bytes, options ? *options : default_options()};
  // a negative chunk_tokens reaches check_common unrounded and is refused there
  const int64_t ct = chunk_tokens < 0 ? chunk_tokens : fused_chunk_tokens(chunk_tokens);
  WsLayout L;
  kdkl_status st = check_common(c, ct, true, L);
  if (st != KDKL_OK) return st;
  if (workspace_bytes < fused_total(L))
    return fail(KDKL_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, fused_total(L));
  if (!loss || !lse || !dHidden || !dW) return fail(KDKL_ERR_NULL, "loss, lse, dHidden and dW must be non-NULL");
  if (!aligned(loss, 4) || !aligned(lse, 4) || (grad_loss && !aligned(grad_loss, 4)))
    return fail(KDKL_ERR_ALIGN, "loss, lse and grad_loss must be 4-byte aligned");
  if (!aligned(dHidden, 16) || !aligned(dW, 16)) return fail(KDKL_ERR_ALIGN, "dHidden and dW must be 16-byte aligned");
  Device dv;
  if ((st = current_device(dv)) != KDKL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (N == 0) {
    if ((e = cudaMemsetAsync(workspace, 0, 256, s)) != cudaSuccess ||
        (e = cudaMemsetAsync(loss, 0, sizeof(float), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(dW, 0, static_cast<size_t>(V) * d * sizeof(float), s)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync");
    return ok();
  }
  if ((st = run_prepass(c, L, s)) != KDKL_OK) return st;

  uint16_t* gbuf = at<uint16_t>(workspace, L.gbuf);
  float* zbuf = at<float>(workspace, fused_logit_offset(L));
  const Pairing pg = pairing(dv.sms, 256);
  const BackwardPlan plan = plan_backward(N, d, V, L.chunk, ct == 0, c.opt.bwd_tile_n, dv.sms);
  const int bn = plan.bn;
  const int64_t chunk = plan.chunk;
  const Pairing pd = pairing(dv.sms, bn);
  CUtensorMap tmW_k, tmW_mn;
  if (!make_map(&tmW_k, W, d, V, d, kBK, pg.b_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tmW_mn, W, d, V, d, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(KDKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (W)");
  const int vt = (V + 255) / 256;
  EpiParams ep0 = base_params(c, L);
  ep0.lse = lse;
  ep0.grad_loss = grad_loss;
  float* part = at<float>(workspace, L.partial);
  const size_t plane = static_cast<size_t>(L.units_cap) * kBM;
  uint32_t* header = at<uint32_t>(workspace, L.header);
  const int64_t total_blocks = (N + 255) / 256;

  for (int64_t c0 = 0; c0 < N; c0 += chunk) {
    const int64_t nc = (N - c0) < chunk ? (N - c0) : chunk;
    const void* hc = static_cast<const uint8_t*>(hidden) + static_cast<size_t>(c0) * d * 2;
    CUtensorMap tmH_k, tmH_mn, tmZ, tmG_k, tmG_mn;
    if (!make_map(&tmH_k, hc, d, nc, d, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmH_mn, hc, d, nc, d, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_f32(&tmZ, zbuf, V, nc, L.Vp, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmG_k, gbuf, V, nc, L.Vp, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmG_mn, gbuf, V, nc, L.Vp, 64, kBK, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(KDKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (chunk maps)");

    // (1) the chunk's logits: online lse + gather partials, and the logits stored
    const int64_t rbc = (nc + pg.rows - 1) / pg.rows;
    const int splits = pick_splits(rbc, vt, pg.groups, d, L.units_cap * kBM / pg.rows, pg.rows);
    {
      Sched sc{static_cast<int>(rbc * splits), splits, vt, (d + kBK - 1) / kBK, kSplitMajor};
      sc.rb_group = split_rb_group(d, pg.rows);
      EpiParams ep = ep0;
      ep.M = static_cast<int>(nc);
      ep.Ncols = V;
      ep.row_offset = c0;
      ep.part_m = part;
      ep.part_s = part + plane;
      ep.part_a = part + 2 * plane;
      ep.part_cap = static_cast<int64_t>(plane);
      const int grid = pg.grid(sc.units);
      if ((e = arm_sync(sc, at<unsigned long long>(workspace, L.sync), grid, pg.pair, s)) != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync");
      if ((e = timed(kTFusedFwd, s, [&] {
             return launch_gemm(kEpiLseStore, 256, pg.pair, tmH_k, tmW_k, tmZ, sc, ep, grid, s);
           })) != cudaSuccess)
        return cuda_fail(e, "fused forward GEMM launch");
    }
    // (2) the chunk's lse and loss terms (the last chunk's last block writes the loss)
    if ((e = timed(kTMerge, s, [&] {
           return launch_merge(part, part + plane, part + 2 * plane, splits, pg.rows, c.opt.student_tau,
                               at<float>(workspace, L.negent) + c0, at<float>(workspace, L.wsum) + c0,
                               at<uint8_t>(workspace, L.rowmask) + c0, nc, lse + c0, loss,
                               at<double>(workspace, L.blocksum), header, ep0.n_valid, c0 / 256, total_blocks,
                               static_cast<int64_t>(plane), s);
         })) != cudaSuccess)
      return cuda_fail(e, "merge launch");
    // (3) G from the stored logits
    if ((e = timed(kTGPass, s, [&] {
           return launch_gpass(zbuf, L.Vp, gbuf, L.Vp, nc, V, c0, ep0.sidx, ep0.sprob, ep0.Kp, ep0.rowmask,
                               ep0.wsum, lse, ep0.n_valid, grad_loss, c.opt.student_tau, ep0.flags, s);
         })) != cudaSuccess)
      return cuda_fail(e, "G launch");
    // (4) dHidden rows of the chunk = G W; (5) dW (+)= G^T hidden_chunk
    if ((st = run_dh_dw(ep0, pd, bn, V, d, c0, nc, tmG_k, tmG_mn, tmW_mn, tmH_mn, dHidden, dW,
                        at<unsigned long long>(workspace, L.sync), s)) != KDKL_OK)
      return st;
  }
  return ok();
}

kdkl_status kdkl_backward(const void* hidden, const void* W, const int32_t* topk_idx, const float* topk_logit,
                          const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau, const float* lse,
                          const float* grad_loss, void* dHidden, float* dW, int64_t chunk_tokens, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return backward_impl(hidden, W, topk_idx, topk_logit, mask, N, d, V, K, tau, nullptr, lse, grad_loss, dHidden, dW,
                       chunk_tokens, workspace, workspace_bytes, stream);
}

kdkl_status kdkl_backward_ex(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                             const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                             const kdkl_options* options, const float* lse, const float* grad_loss, void* dHidden,
                             float* dW, int64_t chunk_tokens, void* workspace, size_t workspace_bytes, void* stream) {
  return backward_impl(hidden, W, topk_idx, topk_logit, mask, N, d, V, K, tau, options, lse, grad_loss, dHidden, dW,
                       chunk_tokens, workspace, workspace_bytes, stream);
}

size_t kdkl_forward_backward_workspace_bytes(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens) {
  if (check_shapes(N, d, V, K, 1.0f) != KDKL_OK || chunk_tokens < 0) return 0;
  return fused_total(make_layout(N, d, V, K, fused_chunk_tokens(chunk_tokens)));
}

kdkl_status kdkl_forward_backward(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                                  const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                                  const kdkl_options* options, const float* grad_loss, float* loss, float* lse,
                                  void* dHidden, float* dW, int64_t chunk_tokens, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return forward_backward_impl(hidden, W, topk_idx, topk_logit, mask, N, d, V, K, tau, options, grad_loss, loss, lse,
                               dHidden, dW, chunk_tokens, workspace, workspace_bytes, stream);
}

void kdkl_options_init(kdkl_options* options) {
  if (options) *options = default_options();
}

kdkl_status kdkl_backward_plan(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens,
                               const kdkl_options* options, int32_t sm_count, int32_t* tile_n_out,
                               int64_t* chunk_tokens_out) {
  if (!tile_n_out || !chunk_tokens_out) return fail(KDKL_ERR_NULL, "tile_n_out and chunk_tokens_out must be non-NULL");
  kdkl_status st = check_shapes(N, d, V, K, 1.0f);
  if (st != KDKL_OK) return st;
  if (chunk_tokens < 0) return fail(KDKL_ERR_SHAPE, "chunk_tokens must be >= 0");
  if (sm_count < 0) return fail(KDKL_ERR_SHAPE, "sm_count must be >= 0");
  const kdkl_options o = options ? *options : default_options();
  if (o.bwd_tile_n != 0 && !pair_tile_n_ok(o.bwd_tile_n))
    return fail(KDKL_ERR_UNSUPPORTED, "bwd_tile_n=%d is not 0 or one of 128, 160, 192, 224, 240, 256", o.bwd_tile_n);
  int sms = sm_count;
  if (sms == 0) {
    Device dv;
    if ((st = current_device(dv)) != KDKL_OK) return st;
    sms = dv.sms;
  }
  const WsLayout L = make_layout(N, d, V, K, chunk_tokens);
  const BackwardPlan plan = plan_backward(N, d, V, L.chunk, chunk_tokens == 0, o.bwd_tile_n, sms);
  *tile_n_out = plan.bn;
  *chunk_tokens_out = plan.chunk;
  return ok();
}

kdkl_status kdkl_count_valid(const void* topk_idx, const void* topk_logit, const uint8_t* mask, int64_t N,
                             int32_t V, int32_t K, float tau, const kdkl_options* options, void* workspace,
                             size_t workspace_bytes, void* stream) {
  // the count needs no hidden states or weights; d only sizes the backward's buffers
  const Common c{nullptr,   nullptr,   topk_idx,        topk_logit, mask, N, 8, V, K, tau,
                 workspace, workspace_bytes, options ? *options : default_options()};
  kdkl_status st = check_shapes(N, 8, V, K, tau);
  if (st != KDKL_OK) return st;
  if (!topk_idx || !topk_logit || !mask || !workspace)
    return fail(KDKL_ERR_NULL, "topk_idx, topk_logit, mask and workspace must be non-NULL");
  if ((st = check_options(c)) != KDKL_OK) return st;
  const size_t cache_align = c.opt.cache_format == KDKL_CACHE_U16_BF16 ? 2 : 4;
  if (!aligned(topk_idx, cache_align) || !aligned(topk_logit, cache_align))
    return fail(KDKL_ERR_ALIGN, "topk_idx and topk_logit must be %zu-byte aligned", cache_align);
  if (!aligned(workspace, 256)) return fail(KDKL_ERR_ALIGN, "workspace must be 256-byte aligned");
  const WsLayout L = make_layout(N, 8, V, K, 0);
  if (workspace_bytes < L.gbuf)
    return fail(KDKL_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.gbuf);
  Device dv;
  if ((st = current_device(dv)) != KDKL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    const cudaError_t e = cudaMemsetAsync(workspace, 0, 256, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    return ok();
  }
  if ((st = run_prepass(c, L, s)) != KDKL_OK) return st;
  return ok();
}

const uint32_t* kdkl_n_valid_device(const void* workspace) {
  return workspace ? reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(workspace) + 4) : nullptr;
}

// ---------------------------------------------------------------- teacher top-K producer
namespace {
struct TopkLayout {
  size_t header = 0, sync = 0, tv = 0, ti = 0, total = 0;
  int s_cap = 1;
};

TopkLayout topk_layout(int64_t N, int32_t K) {
  TopkLayout L;
  L.s_cap = kTopKMergeCand / K > 0 ? kTopKMergeCand / K : 1;
  // enough partial slots for either tile height (256-row pairs or 128-row CTAs)
  const size_t slots = static_cast<size_t>((N + 255) / 256 + 1) * 256 * L.s_cap * K;
  size_t off = 256;
  L.sync = off;
  off += static_cast<size_t>(kSyncSlots) * 8;
  L.tv = off;
  off = align_up(off + slots * 4, 256);
  L.ti = off;
  off = align_up(off + slots * 4, 256);
  L.total = off;
  return L;
}

kdkl_status check_topk_shapes(int64_t N, int32_t d, int32_t V, int32_t K) {
  if (N < 0 || N > kMaxRows) return fail(KDKL_ERR_SHAPE, "N=%lld outside [0, %lld]", (long long)N, (long long)kMaxRows);
  if (d < 8 || d % 8 != 0) return fail(KDKL_ERR_SHAPE, "d=%d must be a positive multiple of 8", d);
  if (V < 1 || V > kMaxV) return fail(KDKL_ERR_SHAPE, "V=%d outside [1, 2^30]", V);
  if (K < 1 || K > kTopKMax || K > V) return fail(KDKL_ERR_SHAPE, "K=%d outside [1, min(%d, V)]", K, kTopKMax);
  // every vocabulary split spans at most kTopKUnitTiles tiles, with at most
  // kTopKMergeCand / K splits
  const int64_t vt = (static_cast<int64_t>(V) + 255) / 256;
  const int64_t s_cap = kTopKMergeCand / K;
  if ((vt + s_cap - 1) / s_cap > kTopKUnitTiles)
    return fail(KDKL_ERR_SHAPE, "V=%d above %lld for K=%d", V, (long long)(kTopKUnitTiles * 256LL * s_cap), K);
  return KDKL_OK;
}
}  // namespace

size_t kdkl_teacher_topk_workspace_bytes(int64_t N, int32_t d, int32_t V, int32_t K) {
  if (check_topk_shapes(N, d, V, K) != KDKL_OK) return 0;
  return topk_layout(N, K).total;
}

kdkl_status kdkl_teacher_topk(const void* hidden, const void* W, int64_t N, int32_t d, int32_t V, int32_t K,
                              int32_t* topk_idx, float* topk_logit, void* workspace, size_t workspace_bytes,
                              void* stream) {
  kdkl_status st = check_topk_shapes(N, d, V, K);
  if (st != KDKL_OK) return st;
  if (!hidden || !W || !topk_idx || !topk_logit || !workspace)
    return fail(KDKL_ERR_NULL, "hidden, W, topk_idx, topk_logit and workspace must be non-NULL");
  if (!aligned(hidden, 16) || !aligned(W, 16)) return fail(KDKL_ERR_ALIGN, "hidden and W must be 16-byte aligned");
  if (!aligned(topk_idx, 4) || !aligned(topk_logit, 4))
    return fail(KDKL_ERR_ALIGN, "topk_idx and topk_logit must be 4-byte aligned");
  if (!aligned(workspace, 256)) return fail(KDKL_ERR_ALIGN, "workspace must be 256-byte aligned");
  const TopkLayout L = topk_layout(N, K);
  if (workspace_bytes < L.total)
    return fail(KDKL_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
  Device dv;
  if ((st = current_device(dv)) != KDKL_OK) return st;
  const Pairing pr = pairing(dv.sms, 256);
  if (!pr.pair) return fail(KDKL_ERR_UNSUPPORTED, "the top-K producer needs CTA pairs");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if ((e = cudaMemsetAsync(workspace, 0, 256, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if (N == 0) return ok();
  const int64_t rb = (N + pr.rows - 1) / pr.rows;
  const int vt = (V + 255) / 256;
  const int splits = pick_splits(rb, vt, pr.groups, d, rb * L.s_cap, pr.rows,
                                 (vt + kTopKUnitTiles - 1) / kTopKUnitTiles);
  Sched sc{static_cast<int>(rb * splits), splits, vt, (d + kBK - 1) / kBK, kRowMajor};
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, hidden, d, N, d, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tmB, W, d, V, d, kBK, pr.b_rows, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(KDKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (hidden/W)");
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.M = static_cast<int>(N);
  ep.Ncols = V;
  ep.topk_K = K;
  ep.part_tv = at<float>(workspace, L.tv);
  ep.part_ti = at<int>(workspace, L.ti);
  ep.topk_cap = static_cast<int64_t>((L.ti - L.tv) / 4);
  ep.flags = at<uint32_t>(workspace, 0);
  ep.exp_scale = 1.4426950408889634f;
  ep.inv_tau_s = 1.0f;
  const int grid = pr.grid(sc.units);
  if ((e = arm_sync(sc, at<unsigned long long>(workspace, L.sync), grid, true, s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync");
  if ((e = timed(kTTopK, s, [&] { return launch_gemm(kEpiTopK, 256, true, tmA, tmB, tmA, sc, ep, grid, s); })) !=
      cudaSuccess)
    return cuda_fail(e, "top-K GEMM launch");
  if ((e = timed(kTTopKMerge, s, [&] {
         return launch_topk_merge(ep.part_tv, ep.part_ti, splits, pr.rows, K, N, topk_idx, topk_logit, ep.topk_cap,
                                  ep.flags, s);
       })) != cudaSuccess)
    return cuda_fail(e, "top-K merge launch");
  return ok();
}

kdkl_status kdkl_selftest_wait_timeout(void* workspace, uint64_t limit_ns, void* stream) {
  if (!workspace) return fail(KDKL_ERR_NULL, "workspace must be non-NULL");
  if (!aligned(workspace, 256)) return fail(KDKL_ERR_ALIGN, "workspace must be 256-byte aligned");
  if (limit_ns < 1000 || limit_ns > 1000000000ull) return fail(KDKL_ERR_SHAPE, "limit_ns outside [1 us, 1 s]");
  Device dv;
  kdkl_status st = current_device(dv);
  if (st != KDKL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, 256, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if ((e = launch_wait_selftest(static_cast<uint32_t*>(workspace),
                                limit_ns, reinterpret_cast<uint64_t*>(static_cast<uint8_t*>(workspace) + 8),
                                s)) != cudaSuccess)
    return cuda_fail(e, "self-test launch");
  return ok();
}

kdkl_status kdkl_timing_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_tmu);
  g_timing = enable != 0;
  return ok();
}

int kdkl_timing_read(kdkl_kernel_time* out, int max_entries, int reset) {
  std::vector<TimingRec> pend;
  {
    std::lock_guard<std::mutex> lk(g_tmu);
    pend.swap(g_pending);
  }
  for (const TimingRec& r : pend) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      std::lock_guard<std::mutex> lk(g_tmu);
      g_launches[r.kind] += 1;
      g_ms[r.kind] += ms;
    }
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  std::lock_guard<std::mutex> lk(g_tmu);
  for (int k = 0; k < kTKinds && k < max_entries && out; ++k) {
    out[k].name = kTimedNames[k];
    out[k].launches = g_launches[k];
    out[k].total_ms = g_ms[k];
  }
  if (reset) {
    for (int k = 0; k < kTKinds; ++k) {
      g_launches[k] = 0;
      g_ms[k] = 0;
    }
  }
  return kTKinds;
}

kdkl_status kdkl_read_device_flags(const void* workspace, void* stream, uint32_t* flags_out) {
  if (!workspace || !flags_out) return fail(KDKL_ERR_NULL, "workspace and flags_out must be non-NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(flags_out, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device flag word");
  return ok();
}

}  // extern "C"
