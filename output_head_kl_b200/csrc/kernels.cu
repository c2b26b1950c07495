// Device kernels of the fused chunked KL loss (sm_100a).
//
//   prepass : per row, sort the cached (index, logit) pairs by index, merge
//             repeats, P_T = softmax(logit / tau), teacher sum P log P,
//             effective mask and N_valid.
//   gemm    : one warp-specialised tcgen05 kernel template (TMA producer warp,
//             MMA warp, four epilogue warps reading TMEM) with four fused
//             epilogues:
//               kEpiLse       forward: running max / sum-exp / gathered logit per row
//               kEpiGrad      backward: recomputed logits -> G chunk (bf16, TMA store)
//               kEpiStoreBf16 dHidden = G W  (fp32 in TMEM, bf16 out)
//               kEpiRmwF32    dW (+)= G^T hidden (fp32 read-modify-write, no atomics)
//   merge   : combine the split-vocabulary partials into lse and the loss
//             (deterministic tree + fixed-order final sum).
//
// Method: the fused chunked KL loss of "Efficient Knowledge Distillation for
// LLMs: Offline Top-K Logits and a Fused Chunked KL Loss" (mind-verse.de
// article, three-variant list, "Fused chunked KL": the projection is folded
// into the loss, chunks are discarded, the backward recomputes them; llm-wiki
// note, section "Fused Chunked KL": softmax, log and KL fused in one kernel).
#include <cfloat>
#include <climits>
#include <cmath>

#include <atomic>

#include "kdkl_internal.h"
#include "sm100.cuh"

namespace kdkl {

constexpr float kLog2e = 1.4426950408889634f;

// ============================================================================
// prepass: one warp per row
//
// Builds each row's target list: the teacher's cached entries with indices
// outside [0, V) dropped, sorted by index, repeats merged, probabilities
// gamma * softmax(logit / tau), plus beta at the row's hard label when one is
// given (merged into the cached entry of the same index, or inserted).  Also
// writes gamma * sum P_T log P_T, the list's total weight, the effective mask,
// N_valid and the data-error flags.
// ============================================================================
constexpr int kPreWarps = 8;
constexpr int kListMax = kMaxK + 4;   // cached entries + the label, with room to spare

__device__ __forceinline__ int load_idx(const int32_t* p, int64_t i) { return p[i]; }
__device__ __forceinline__ int load_idx(const uint16_t* p, int64_t i) { return static_cast<int>(p[i]); }
__device__ __forceinline__ float load_logit(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_logit(const uint16_t* p, int64_t i) {
  return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);   // bf16 -> fp32, exact
}

template <typename IdxT, typename LogitT>
__global__ void __launch_bounds__(kPreWarps * 32)
    prepass_kernel(const IdxT* __restrict__ topk_idx, const LogitT* __restrict__ topk_logit,
                   const uint8_t* __restrict__ mask, const int32_t* __restrict__ labels, int64_t N, int V, int K,
                   float inv_tau, float gamma, float beta, int* __restrict__ sidx, float* __restrict__ sprob,
                   float* __restrict__ negent, float* __restrict__ wsum, uint8_t* __restrict__ rowmask, int Kp,
                   uint32_t* __restrict__ header) {
  __shared__ int s_key[kPreWarps][kListMax];
  __shared__ float s_p[kPreWarps][kListMax];
  __shared__ int s_skey[kPreWarps][kListMax];
  __shared__ float s_sp[kPreWarps][kListMax];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* key = s_key[w];
  float* pv = s_p[w];
  int* skey = s_skey[w];
  float* sp = s_sp[w];
  uint32_t wflags = 0;
  uint32_t wvalid = 0;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * kPreWarps;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * kPreWarps + w; n < N; n += warps_total) {
    const int64_t base_in = n * K;
    int ki[8];
    float xi[8];
    bool keep[8];
    bool any_keep = false, any_bad = false, any_drop = false;
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane + 32 * i;
      ki[i] = 0;
      xi[i] = -INFINITY;
      keep[i] = false;
      if (k < K) {
        const int id = load_idx(topk_idx, base_in + k);
        const float x = load_logit(topk_logit, base_in + k) * inv_tau;
        keep[i] = (id >= 0) && (id < V);
        ki[i] = id;
        xi[i] = x;
        if (!keep[i]) any_drop = true;
        if (keep[i]) {
          any_keep = true;
          if (isnan(x) || x == INFINITY) any_bad = true;
          else mx = fmaxf(mx, x);
        }
      }
    }
    any_keep = __any_sync(0xffffffffu, any_keep);
    any_bad = __any_sync(0xffffffffu, any_bad);
    any_drop = __any_sync(0xffffffffu, any_drop);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (any_drop) wflags |= 1u;
    const bool row_ok = any_keep && !any_bad && (mx > -INFINITY);
    if (any_keep && !row_ok) wflags |= 4u;
    int* out_i = sidx + n * Kp;
    float* out_p = sprob + n * Kp;
    if (!row_ok) {
      for (int k = lane; k < Kp; k += 32) {
        out_i[k] = kSentinel;
        out_p[k] = 0.f;
      }
      if (lane == 0) {
        negent[n] = 0.f;
        wsum[n] = 0.f;
        rowmask[n] = 0;
      }
      __syncwarp();
      continue;
    }
    // teacher probabilities over the in-range entries
    float e[8];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      e[i] = keep[i] ? expf(xi[i] - mx) : 0.f;
      sum += e[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.f / sum;
    // sort keys: in-range entries by index, dropped entries after them (key V + k)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane + 32 * i;
      if (k < K) {
        key[k] = keep[i] ? ki[i] : (V + k);
        pv[k] = e[i] * inv;
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane + 32 * i;
      if (k < K) {
        const int mine = key[k];
        int rank = 0;
        for (int j = 0; j < K; ++j) {
          const int other = key[j];
          rank += (other < mine) || (other == mine && j < k);
        }
        if (dbg_ok(rank < K, header)) {
          skey[rank] = mine;
          sp[rank] = pv[k];
        }
      }
    }
    __syncwarp();
    // merge runs of equal indices, compact into key/pv, and sum P log P
    float ent = 0.f;
    int cnt = 0;
    bool dup = false;
    for (int r0 = 0; r0 < K; r0 += 32) {
      const int r = r0 + lane;
      bool start = false;
      float pm = 0.f;
      int kk = kSentinel;
      if (r < K) {
        kk = skey[r];
        if (kk < V) {
          start = (r == 0) || (skey[r - 1] != kk);
          if (!start) dup = true;
          if (start) {
            pm = sp[r];
            for (int t = r + 1; t < K && skey[t] == kk; ++t) pm += sp[t];
          }
        }
      }
      const uint32_t ballot = __ballot_sync(0xffffffffu, start);
      const int pos = cnt + __popc(ballot & ((1u << lane) - 1u));
      if (start && dbg_ok(pos < Kp - 1, header)) {   // room for the sentinel after the list
        key[pos] = kk;
        pv[pos] = gamma * pm;
        if (pm > 0.f) ent += pm * logf(pm);
      }
      cnt += __popc(ballot);
    }
    __syncwarp();
    // the hard label joins the list with weight beta
    float wrow = gamma;
    if (labels != nullptr && beta != 0.f) {
      const int lab = labels[n];
      if (lab >= 0 && lab < V) {
        wrow += beta;
        int grew = 0;
        if (lane == 0) {
          int lo = 0, hi = cnt;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (key[mid] < lab) lo = mid + 1;
            else hi = mid;
          }
          if (lo < cnt && key[lo] == lab) {
            pv[lo] += beta;
          } else if (dbg_ok(cnt + 1 < Kp, header)) {
            for (int t = cnt; t > lo; --t) {
              key[t] = key[t - 1];
              pv[t] = pv[t - 1];
            }
            key[lo] = lab;
            pv[lo] = beta;
            grew = 1;
          }
        }
        cnt += __shfl_sync(0xffffffffu, grew, 0);
        __syncwarp();
      }
    }
    for (int k = lane; k < Kp; k += 32) {
      out_i[k] = k < cnt ? key[k] : kSentinel;
      out_p[k] = k < cnt ? pv[k] : 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ent += __shfl_xor_sync(0xffffffffu, ent, o);
    if (__any_sync(0xffffffffu, dup)) wflags |= 2u;
    if (lane == 0) {
      negent[n] = gamma * ent;
      wsum[n] = wrow;
      const uint8_t m = (mask[n] != 0) ? 1 : 0;
      rowmask[n] = m;
      wvalid += m;
    }
    __syncwarp();
  }
  if (lane == 0) {
    if (wflags) atomicOr(&header[0], wflags);
    if (wvalid) atomicAdd(&header[1], wvalid);
  }
}

cudaError_t launch_prepass(int cache_format, const void* topk_idx, const void* topk_logit, const uint8_t* mask,
                           const int32_t* labels, int64_t N, int32_t V, int32_t K, float tau, float gamma,
                           float beta, int* sidx, float* sprob, float* negent, float* wsum, uint8_t* rowmask,
                           int Kp, uint32_t* header, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (N + kPreWarps - 1) / kPreWarps;
  const int grid = static_cast<int>(want < static_cast<int64_t>(sms) * 8 ? want : static_cast<int64_t>(sms) * 8);
  if (cache_format == 1)
    prepass_kernel<uint16_t, uint16_t><<<grid, kPreWarps * 32, 0, stream>>>(
        static_cast<const uint16_t*>(topk_idx), static_cast<const uint16_t*>(topk_logit), mask, labels, N, V, K,
        1.0f / tau, gamma, beta, sidx, sprob, negent, wsum, rowmask, Kp, header);
  else
    prepass_kernel<int32_t, float><<<grid, kPreWarps * 32, 0, stream>>>(
        static_cast<const int32_t*>(topk_idx), static_cast<const float*>(topk_logit), mask, labels, N, V, K,
        1.0f / tau, gamma, beta, sidx, sprob, negent, wsum, rowmask, Kp, header);
  return cudaGetLastError();
}

// ============================================================================
// merge: split-vocabulary partials -> lse, per-row KL, loss
// ============================================================================
constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
    merge_kernel(const float* __restrict__ part_m, const float* __restrict__ part_s,
                 const float* __restrict__ part_a, int splits, int rows_per_block, float inv_tau_s,
                 const float* __restrict__ negent, const float* __restrict__ wsum,
                 const uint8_t* __restrict__ rowmask, int64_t N, float* __restrict__ lse,
                 float* __restrict__ loss, double* __restrict__ blocksum, uint32_t* __restrict__ header,
                 const uint32_t* __restrict__ n_valid, int64_t block_base, int64_t total_blocks,
                 int64_t part_cap) {
  __shared__ double s_red[kMergeThreads / 32];
  __shared__ bool s_last;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kMergeThreads + threadIdx.x;
  double kl = 0.0;
  const int64_t rb = n / rows_per_block;
  if (n < N && dbg_ok((rb * splits + splits) * rows_per_block <= part_cap, header)) {
    const int r = static_cast<int>(n - rb * rows_per_block);
    float M = -INFINITY;
    for (int j = 0; j < splits; ++j) M = fmaxf(M, part_m[(rb * splits + j) * rows_per_block + r]);
    float s = 0.f, a = 0.f;
    for (int j = 0; j < splits; ++j) {
      const int64_t slot = (rb * splits + j) * rows_per_block + r;
      s += part_s[slot] * expf((part_m[slot] - M) * inv_tau_s);
      a += part_a[slot];
    }
    // lse of z / tau_s; the row's loss is gamma sum P_T log P_T - sum target * z / tau_s + weight * lse
    const float l = M * inv_tau_s + logf(s);
    lse[n] = l;
    if (rowmask[n])
      kl = static_cast<double>(negent[n]) - static_cast<double>(a) * inv_tau_s +
           static_cast<double>(wsum[n]) * static_cast<double>(l);
  }
  // block tree reduction (fixed order)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kl += __shfl_xor_sync(0xffffffffu, kl, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = kl;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < kMergeThreads / 32; ++i) t += s_red[i];
    blocksum[block_base + blockIdx.x] = t;
    __threadfence();
    const uint32_t ticket = atomicAdd(&header[2], 1u);
    s_last = (static_cast<int64_t>(ticket) == total_blocks - 1);
  }
  __syncthreads();
  if (s_last && threadIdx.x == 0) {
    __threadfence();
    double t = 0.0;
    const volatile double* bs = blocksum;
    for (int64_t i = 0; i < total_blocks; ++i) t += bs[i];
    const uint32_t nv = *reinterpret_cast<const volatile uint32_t*>(n_valid);
    loss[0] = nv > 0 ? static_cast<float>(t / static_cast<double>(nv)) : 0.f;
    header[2] = 0;
  }
}

cudaError_t launch_merge(const float* part_m, const float* part_s, const float* part_a, int splits,
                         int rows_per_block, float student_tau, const float* negent, const float* wsum,
                         const uint8_t* rowmask, int64_t N, float* lse, float* loss, double* blocksum,
                         uint32_t* header, const uint32_t* n_valid, int64_t block_base, int64_t total_blocks,
                         int64_t part_cap, cudaStream_t stream) {
  const int grid = static_cast<int>((N + kMergeThreads - 1) / kMergeThreads);
  if (total_blocks <= 0) total_blocks = grid;
  merge_kernel<<<grid, kMergeThreads, 0, stream>>>(part_m, part_s, part_a, splits, rows_per_block,
                                                   1.0f / student_tau, negent, wsum, rowmask, N, lse, loss,
                                                   blocksum, header, n_valid, block_base, total_blocks, part_cap);
  return cudaGetLastError();
}

// ============================================================================
// warp-specialised tcgen05 GEMM with fused epilogues
//
// PAIR = false: one CTA computes a 128 x BN tile (M = 128 MMAs, cta_group::1).
// PAIR = true : a cluster of two CTAs computes a 256 x BN tile with M = 256
//               MMAs issued by the even CTA (cta_group::2).  Each CTA loads
//               its own 128 rows of A and half (BN/2 rows) of B, so per flop
//               each SM streams a third less operand data from L2 and reads a
//               third less from shared memory.  Each CTA's TMEM holds the
//               accumulator rows of its own 128 rows; both epilogues run in
//               parallel, one per CTA.
// ============================================================================
template <int KIND, int BN, bool PAIR>
struct GemmCfg {
  static constexpr bool kAmn = (KIND == kEpiRmwF32);
  static constexpr bool kBmn = (KIND == kEpiStoreBf16 || KIND == kEpiRmwF32);
  static constexpr int kCtaN = PAIR ? BN / 2 : BN;     // B rows (N) held by this CTA
  static constexpr int kMmaM = PAIR ? 256 : 128;       // rows of one tile across the pair
  // An MN-major B is staged as whole 64-column swizzle atoms; when kCtaN is not a
  // multiple of 64 the MMA reads only the first kCtaN columns of the last atom
  // (the rest is in-bounds neighbour data or TMA zero fill).
  static constexpr int kBAtoms = (kCtaN + 63) / 64;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = kBmn ? kBAtoms * 64 * kBK * 2 : kCtaN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;               // landing in this CTA
  static constexpr int kTxBytes = (PAIR ? 2 : 1) * kStageBytes;       // counted on the MMA's barrier
  // per-epilogue-warp staging: grad 2 x 2 KB (32 x 32 bf16), dW 4 KB (32 x 32 fp32),
  // stored logits 2 x 4 KB (32 x 32 fp32); top-K: the heaps of all 128 rows
  // dW: 2 x 4 KB (32 x 32 fp32, the old block loaded and the new one stored through it)
  static constexpr int kEpiWarpBytes = (KIND == kEpiLseStore || KIND == kEpiRmwF32) ? 8192 : 4096;
  static constexpr int kEpiBytes = (KIND == kEpiGrad || KIND == kEpiRmwF32 || KIND == kEpiLseStore)
                                       ? 4 * kEpiWarpBytes
                                       : (KIND == kEpiTopK ? kTopKMax * kBM * 6 : 0);
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemLimit = 232448;
  static constexpr int kStagesFit = (kSmemLimit - 1024 - kEpiBytes - kBarBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kEpiBytes + kBarBytes;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kMmaM, BN, kAmn, kBmn);
  // the two accumulators sit at TMEM columns 0 and kAccStride (a power of two >= BN)
  static constexpr int kAccStride = BN <= 128 ? 128 : 256;
  static constexpr uint32_t kTmemCols = (2 * kAccStride <= 256) ? 256u : 512u;
  static constexpr int kAccEmptyArrivals = PAIR ? 8 : 4;
  // tcgen05.mma kind::f16 with both operands in shared memory: N a multiple of 16 in
  // [16, 256] for cta_group::2 (M = 256) and cta_group::1 (M = 128); BN % 16 also keeps
  // each CTA's B coordinate (rank * kCtaN) on the 16-byte TMA boundary
  static_assert(BN % 16 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(BN % 32 == 0 || KIND == kEpiStoreBf16 || KIND == kEpiRmwF32,
                "the loss epilogues read whole 32-column TMEM chunks of a tile");
  static_assert(kStages >= 2, "stages");
};

// Unit u -> row block mb, vocabulary split j (row-stream units; 0 otherwise) and
// its tile range [t0, t1).
__device__ __forceinline__ void unit_range(const Sched& sc, int u, int& mb, int& j, int& t0, int& t1) {
  j = 0;
  if (sc.row_stream) {
    if (sc.row_stream == kSplitMajor) {
      // groups of rb_group row blocks, each swept split by split; the last group may
      // hold fewer row blocks
      const int rb = sc.units / sc.splits;
      const int gsz = (sc.rb_group > 0 && sc.rb_group < rb) ? sc.rb_group : rb;
      const int g = u / (gsz * sc.splits);
      const int rbg = min(gsz, rb - g * gsz);
      const int off = u - g * gsz * sc.splits;
      j = off / rbg;
      mb = g * gsz + (off - j * rbg);
    } else {
      mb = u / sc.splits;
      j = u - mb * sc.splits;
    }
    t0 = static_cast<int>((static_cast<int64_t>(j) * sc.n_tiles) / sc.splits);
    t1 = static_cast<int>((static_cast<int64_t>(j + 1) * sc.n_tiles) / sc.splits);
  } else {
    // groups of col_group column tiles (0 = all), each swept row block by row block;
    // the last group may hold fewer tiles
    const int rows = sc.units / sc.n_tiles;
    const int cg = (sc.col_group > 0 && sc.col_group < sc.n_tiles) ? sc.col_group : sc.n_tiles;
    const int g = u / (rows * cg);
    const int cgs = min(cg, sc.n_tiles - g * cg);
    const int off = u - g * rows * cg;
    mb = off / cgs;
    t0 = g * cg + (off - mb * cgs);
    t1 = t0 + 1;
  }
}

// Position word a group publishes as it reaches position r of unit u (the relative tile
// of a row-stream unit, the reduction block of a tile-mode unit).
__device__ __forceinline__ unsigned long long sync_word(int u, int r) {
  return (static_cast<unsigned long long>(u + 1) << 32) | static_cast<unsigned int>(r);
}

// Whole warp (the producer warp of an even CTA): the smallest position that the peers
// of unit u have reached in their units (a peer already past its unit counts as
// INT_MAX, one not yet in it as -1), waiting until it is at least r_need.  The peers
// are the other units of u's round that stream the same operand: those of vocabulary
// split j (row-stream launches), or every unit of the round (tile-mode launches, whose
// units share rows of A or columns of B).  Returns -2 if the wait gave up
// (kSyncSoftLimitNs).
__device__ int wait_split_peers(const Sched& sc, int u, int group, int ngroups, int j, int r_need, int lane,
                                uint32_t* flags) {
  const int round0 = u - group;                  // group g runs units g + k G: this round is [k G, k G + G)
  const int round1 = min(round0 + ngroups, sc.units);
  int first, last, step;
  if (sc.row_stream == 0) {                      // tile mode: the whole round
    first = round0;
    last = round1;
    step = 1;
  } else if (sc.row_stream == kSplitMajor) {     // split j of u's row-block group: contiguous units
    const int rb = sc.units / sc.splits;
    const int gsz = (sc.rb_group > 0 && sc.rb_group < rb) ? sc.rb_group : rb;
    const int g = u / (gsz * sc.splits);
    const int rbg = min(gsz, rb - g * gsz);
    const int gbase = g * gsz * sc.splits;
    first = max(round0, gbase + j * rbg);
    last = min(round1, gbase + (j + 1) * rbg);
    step = 1;
  } else {                                       // units of split j are those with u % splits == j
    first = round0 + ((j - round0 % sc.splits) % sc.splits + sc.splits) % sc.splits;
    last = round1;
    step = sc.splits;
  }
  const uint64_t t0 = globaltimer_ns();
  int seen = INT_MAX;
  for (int base = first; base < last; base += 32 * step) {
    const int up = base + lane * step;
    const bool mine = up < last && up != u;
    const volatile unsigned long long* slot =
        sc.prog + ((mine && dbg_ok(up - round0 < ngroups && ngroups <= kSyncSlots, flags)) ? up - round0 : 0);
    int rel = INT_MAX;
    while (true) {
      if (mine) {
        const unsigned long long w = *slot;
        const unsigned long long hi = w >> 32, want = static_cast<unsigned long long>(up + 1);
        rel = hi > want ? INT_MAX : (hi == want ? static_cast<int>(w & 0xFFFFFFFFull) : -1);
      }
      const int lo = __reduce_min_sync(0xffffffffu, rel);
      if (lo >= r_need) {
        seen = min(seen, lo);
        break;
      }
      if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > kSyncSoftLimitNs)) return -2;
      __nanosleep(128);
    }
  }
  return seen;
}

// z[off] for a run-time off in [0, 32) without dynamic register indexing.
// Role cycle counters of the profiling build (-DKDKL_PROFILE).  Each GEMM CTA adds, under
// its epilogue kind, how many SM cycles its TMA producer, its MMA issuer (the even CTA of
// a pair) and its first epilogue warp spent in the kernel and waiting at their barriers:
//   slots 0-3   MMA issuer: total, waiting for a free accumulator, waiting for operands, tiles
//   slots 4-7   producer:   total, waiting for a free stage, waiting in the lockstep, units
//   slots 8-11  epilogue:   total, waiting for a finished accumulator, 0, tiles
// In every other build RoleClock is empty and compiles to nothing.
#if defined(KDKL_PROFILE)
__device__ unsigned long long g_role_cycles[kRoleKinds][kRoleCtas][kRoleSlots];

__device__ __forceinline__ long long sm_cycles() {
#if defined(__CUDA_ARCH__)
  return clock64();
#else
  return 0;
#endif
}

struct RoleClock {
  long long start, w0 = 0, w1 = 0, n = 0;
  __device__ RoleClock() : start(sm_cycles()) {}
  __device__ long long now() const { return sm_cycles(); }
  __device__ void wait0(long long t) { w0 += sm_cycles() - t; }
  __device__ void wait1(long long t) { w1 += sm_cycles() - t; }
  __device__ void count() { ++n; }
  __device__ void flush(int kind, int base) const {
    if (blockIdx.x >= static_cast<unsigned>(kRoleCtas) || kind >= kRoleKinds) return;
    unsigned long long* p = g_role_cycles[kind][blockIdx.x] + base;
    atomicAdd(p + 0, static_cast<unsigned long long>(sm_cycles() - start));
    atomicAdd(p + 1, static_cast<unsigned long long>(w0));
    atomicAdd(p + 2, static_cast<unsigned long long>(w1));
    atomicAdd(p + 3, static_cast<unsigned long long>(n));
  }
};
#else
struct RoleClock {
  __device__ long long now() const { return 0; }
  __device__ void wait0(long long) {}
  __device__ void wait1(long long) {}
  __device__ void count() {}
  __device__ void flush(int, int) const {}
};
#endif

__device__ __forceinline__ float pick32(const float (&v)[32], uint32_t off) {
  float t16[16], t8[8], t4[4], t2[2];
  const bool b4 = off & 16u, b3 = off & 8u, b2 = off & 4u, b1 = off & 2u, b0 = off & 1u;
#pragma unroll
  for (int j = 0; j < 16; ++j) t16[j] = b4 ? v[j + 16] : v[j];
#pragma unroll
  for (int j = 0; j < 8; ++j) t8[j] = b3 ? t16[j + 8] : t16[j];
#pragma unroll
  for (int j = 0; j < 4; ++j) t4[j] = b2 ? t8[j + 4] : t8[j];
#pragma unroll
  for (int j = 0; j < 2; ++j) t2[j] = b1 ? t4[j + 2] : t4[j];
  return b0 ? t2[1] : t2[0];
}

// First position of a sorted, sentinel-terminated list whose value is >= v.
__device__ __forceinline__ int lower_bound_list(const int* __restrict__ lst, int Kp, int v) {
  int lo = 0, hi = Kp - 1;  // lst[Kp - 1] is always the sentinel
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (lst[mid] < v) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

template <int KIND, int BN, bool PAIR>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmOut, const Sched sc, const EpiParams ep) {
  using C = GemmCfg<KIND, BN, PAIR>;
  constexpr bool kLseLike = (KIND == kEpiLse || KIND == kEpiLseStore);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint8_t* sEpi = sB + C::kStages * C::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + C::kEpiBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* acc_full = bars + 2 * C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* ebar = drain + 1;             // dW epilogue: one load barrier per staging buffer (4 warps x 2)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ebar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_group = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // 0 = the CTA that issues the MMAs
  const int ngroups = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::kAccEmptyArrivals);
    }
    mbar_init(drain, 1);
    for (int b = 0; b < 8; ++b) mbar_init(&ebar[b], 1);
    *abort_flag = 0;
    int g = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    if (sc.die_order && rank == 0) {
      // Group numbers by die: the groups on the SMs of the lower half of the SM ids take
      // tickets from 0 upwards, the others from ngroups - 1 downwards, so each half
      // runs a contiguous range of every round's units.  Exactly ngroups groups take one
      // ticket each, so the two ranges meet without overlap whatever the halves' sizes.
      const int die = 2 * static_cast<int>(sm_id()) >= static_cast<int>(sm_count_ids()) ? 1 : 0;
      const unsigned long long t = atomicAdd(sc.prog + ngroups + die, 1ull);
      const int tk = static_cast<int>(t);
      const int gd = die ? ngroups - 1 - tk : tk;
      if (dbg_ok(gd >= 0 && gd < ngroups, ep.flags)) g = gd;
    }
    *s_group = g;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (KIND == kEpiGrad || KIND == kEpiLseStore || KIND == kEpiRmwF32) tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (PAIR) cluster_sync();   // the even CTA's barriers are initialised before any peer signal
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the pair's group number: the even CTA's (read across the cluster by the odd CTA)
  const int group = (PAIR && rank != 0) ? ld_shared_cluster_s32(mapa_shared(smem_u32(s_group), 0)) : *s_group;
  const AbortState ab{abort_flag, ep.flags};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 issues the copies; the whole warp takes part in the lockstep wait.
    int stage = 0;
    uint32_t phase = 0;
    bool wrapped = false;    // every stage has been filled at least once
    RoleClock rc;
    bool stop = false;
    const bool sync_on = sc.sync_window > 0 && rank == 0;
    // row-stream units synchronise per tile; tile-mode units (one long reduction each)
    // per segment of kSyncKStep reduction blocks
    const int kseg = (sync_on && sc.row_stream == 0) ? kSyncKStep : sc.k_blocks;
    const bool hints = (sc.l2_a | sc.l2_b) != 0;
    const uint64_t pol_a = l2_policy(sc.l2_a), pol_b = l2_policy(sc.l2_b);
    for (int u = group; u < sc.units && !stop; u += ngroups) {
      int mb, uj, t0, t1;
      unit_range(sc, u, mb, uj, t0, t1);
      rc.count();
      const int arow = mb * C::kMmaM + static_cast<int>(rank) * kBM;   // this CTA's A rows
      bool hold = sync_on;
      int seen = -1;          // every peer had reached this position at the last look
      for (int t = t0; t < t1 && !stop; ++t) {
        int bcol = t * BN + static_cast<int>(rank) * C::kCtaN;  // this CTA's B rows (N)
        if (C::kBmn && !dbg_ok((bcol & 7) == 0, ep.flags)) bcol &= ~7;   // x of an MN-major bf16 box
        for (int kb0 = 0; kb0 < sc.k_blocks && !stop; kb0 += kseg) {
          if (sync_on) {
            // publish first, then wait: every peer has then published at least the
            // position it waits at, so the slowest peer's condition always holds
            const int pos = sc.row_stream ? t - t0 : kb0;
            const int need = pos - sc.sync_window;
            if (lane == 0) *reinterpret_cast<volatile unsigned long long*>(sc.prog + group) = sync_word(u, pos);
            __syncwarp();
            if (hold && need > seen) {
              const long long c0 = rc.now();
              const int got = wait_split_peers(sc, u, group, ngroups, uj, need, lane, ep.flags);
              rc.wait1(c0);
              if (got == -2) hold = false;
              else seen = got;
            }
          }
          int lstop = 0;
          if (lane == 0) {
            const int kb1 = min(kb0 + kseg, sc.k_blocks);
            for (int kb = kb0; kb < kb1; ++kb) {
              const long long c0 = rc.now();
              const bool got_stage = mbar_wait(&empty[stage], phase ^ 1u, ab);
              rc.wait0(c0);
              if (!got_stage) {
                lstop = 1;
                break;
              }
              uint8_t* a = sA + stage * C::kABytes;
              uint8_t* b = sB + stage * C::kBBytes;
              if (PAIR) {
                // both CTAs' bytes are counted on the even CTA's barrier
                const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
                if (rank == 0) mbar_arrive_expect_tx(&full[stage], C::kTxBytes);
                if (hints) {
                  if (C::kAmn) {
                    tma_load_2d_pair_hint(a, &tmA, bar0, arow, kb * kBK, pol_a);
                    tma_load_2d_pair_hint(a + 8192, &tmA, bar0, arow + 64, kb * kBK, pol_a);
                  } else {
                    tma_load_2d_pair_hint(a, &tmA, bar0, kb * kBK, arow, pol_a);
                  }
                  if (C::kBmn) {
#pragma unroll
                    for (int q = 0; q < C::kBAtoms; ++q)
                      tma_load_2d_pair_hint(b + q * 8192, &tmB, bar0, bcol + q * 64, kb * kBK, pol_b);
                  } else {
                    tma_load_2d_pair_hint(b, &tmB, bar0, kb * kBK, bcol, pol_b);
                  }
                } else {
                  if (C::kAmn) {
                    tma_load_2d_pair(a, &tmA, bar0, arow, kb * kBK);
                    tma_load_2d_pair(a + 8192, &tmA, bar0, arow + 64, kb * kBK);
                  } else {
                    tma_load_2d_pair(a, &tmA, bar0, kb * kBK, arow);
                  }
                  if (C::kBmn) {
#pragma unroll
                    for (int q = 0; q < C::kBAtoms; ++q)
                      tma_load_2d_pair(b + q * 8192, &tmB, bar0, bcol + q * 64, kb * kBK);
                  } else {
                    tma_load_2d_pair(b, &tmB, bar0, kb * kBK, bcol);
                  }
                }
              } else {
                mbar_arrive_expect_tx(&full[stage], C::kTxBytes);
                if (C::kAmn) {
                  tma_load_2d(a, &tmA, &full[stage], arow, kb * kBK);
                  tma_load_2d(a + 8192, &tmA, &full[stage], arow + 64, kb * kBK);
                } else {
                  tma_load_2d(a, &tmA, &full[stage], kb * kBK, arow);
                }
                if (C::kBmn) {
#pragma unroll
                  for (int q = 0; q < C::kBAtoms; ++q)
                    tma_load_2d(b + q * 8192, &tmB, &full[stage], bcol + q * 64, kb * kBK);
                } else {
                  tma_load_2d(b, &tmB, &full[stage], kb * kBK, bcol);
                }
              }
              if (++stage == C::kStages) {
                stage = 0;
                phase ^= 1u;
                wrapped = true;
              }
            }
          }
          stop = __shfl_sync(0xffffffffu, lstop, 0) != 0;
        }
      }
    }
    if (lane == 0) rc.flush(KIND, 4);
    if (lane == 0 && rank == 0 && *abort_flag) {
      // The kernel is giving up: before shared memory is released, wait (bounded) until
      // the copies already issued have landed.  The even CTA's full barriers count
      // both CTAs' bytes, so the last issued phase of each stage covers the pair.
      const uint64_t w0 = globaltimer_ns();
      for (int s2 = 0; s2 < C::kStages; ++s2) {
        if (!wrapped && s2 >= stage) break;              // never filled
        const uint32_t par = s2 < stage ? phase : (phase ^ 1u);
        const uint32_t a = smem_u32(&full[s2]);
        while (!mbar_try_wait(a, par) && globaltimer_ns() - w0 < kDrainLimitNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      RoleClock rc;
      for (int u = group; u < sc.units; u += ngroups) {
        int mb, uj, t0, t1;
        unit_range(sc, u, mb, uj, t0, t1);
        for (int t = t0; t < t1; ++t) {
          const long long c0 = rc.now();
          const bool got_acc = mbar_wait(&acc_empty[acc], acc_phase ^ 1u, ab);
          rc.wait0(c0);
          rc.count();
          if (!got_acc) goto mma_done;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccStride);
          for (int kb = 0; kb < sc.k_blocks; ++kb) {
            const long long c1 = rc.now();
            const bool got_ops = mbar_wait(&full[stage], phase, ab);
            rc.wait1(c1);
            if (!got_ops) goto mma_done;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + stage * C::kABytes);
            const uint32_t b_addr = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
            for (int j = 0; j < kBK / 16; ++j) {
              const uint64_t ad = C::kAmn ? sdesc_sw128(a_addr + j * 2048, 8192, 1024)
                                          : sdesc_sw128(a_addr + j * 32, 16, 1024);
              const uint64_t bd = C::kBmn ? sdesc_sw128(b_addr + j * 2048, 8192, 1024)
                                          : sdesc_sw128(b_addr + j * 32, 16, 1024);
              if (PAIR) umma_bf16_pair(d_tmem, ad, bd, C::kIdesc, (kb | j) != 0 ? 1u : 0u);
              else umma_bf16(d_tmem, ad, bd, C::kIdesc, (kb | j) != 0 ? 1u : 0u);
            }
            if (PAIR) umma_commit_pair(&empty[stage], 0x3);
            else umma_commit(&empty[stage]);
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (PAIR) umma_commit_pair(&acc_full[acc], 0x3);
          else umma_commit(&acc_full[acc]);
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        }
      }
    mma_done:
      rc.flush(KIND, 0);
      // every MMA issued above has finished before TMEM or shared memory is released
      if (PAIR) umma_commit_pair(drain, 0x1);
      else umma_commit(drain);
      {
        const uint32_t a = smem_u32(drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, 0)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(ep.flags, kFlagTimeout);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t acc_empty0 = PAIR ? mapa_shared(smem_u32(&acc_empty[0]), 0) : 0u;
    int acc = 0;
    uint32_t acc_phase = 0;
    float g_scale = 0.f;
    RoleClock rc;
    if (KIND == kEpiGrad) {
      // d loss / d z = (g / (tau_s N_valid)) (weight P_S - target)
      const uint32_t nv = *ep.n_valid;
      const float g = ep.grad_loss ? *ep.grad_loss : 1.0f;
      g_scale = nv > 0 ? g * ep.inv_tau_s / static_cast<float>(nv) : 0.f;
    }
    const float es = ep.exp_scale;   // log2(e) / tau_s
    uint8_t* wbuf = sEpi + (warp - 2) * C::kEpiWarpBytes;   // this warp's staging
    uint8_t* wbuf_all = sEpi;                    // top-K heaps of all 128 rows
    int sbuf = 0;
    // dW: staging buffer of the next TMA chunk, load-barrier phase bits and loads in flight
    uint64_t* wbar = ebar + 2 * (warp - 2);
    uint32_t dw_phase = 0, dw_pending = 0;
    for (int u = group; u < sc.units; u += ngroups) {
      int mb, uj, t0, t1;
      unit_range(sc, u, mb, uj, t0, t1);
      // this unit's partial-result slot: (row block, split) in row-major order, whatever
      // order the units are dealt in (the merges read them that way)
      const int64_t uslot = static_cast<int64_t>(mb) * sc.splits + uj;
      const int row0 = mb * C::kMmaM + static_cast<int>(rank) * kBM;   // first row of this CTA
      const int row = row0 + row_local;
      const bool rv = row < ep.M;
      // teacher top-K: this thread's row owns column row_local of two [kTopKMax][128]
      // shared arrays holding a min-heap ordered by (value, then larger index first).
      // Indices are kept relative to the unit's first column: a unit spans at most
      // kTopKUnitTiles tiles, so 16 bits hold them and kTopKEmpty marks an empty slot
      // (it also ranks after every real index, as the absolute sentinel does).
      float* hv = reinterpret_cast<float*>(wbuf_all) + row_local;
      uint16_t* hi = reinterpret_cast<uint16_t*>(wbuf_all + kTopKMax * kBM * 4) + row_local;
      const int ubase = t0 * BN;
      float hroot = -INFINITY;
      int hcnt = 0;   // entries kept so far (the heap fills before its root becomes a threshold)
      if (KIND == kEpiTopK) {
        for (int k = 0; k < ep.topk_K; ++k) {
          hv[k * kBM] = -INFINITY;
          hi[k * kBM] = kTopKEmpty;
        }
      }
      const int64_t grow = ep.row_offset + row;
      // per-row state of the loss epilogues
      float m_run = -INFINITY, s_run = 0.f, a_run = 0.f;
      float cn = 0.f, cnw = 0.f, lse_l2 = INFINITY;
      int kpos = 0, nxt = kSentinel;
      float nxtp = 0.f;
      const int* lst = nullptr;
      const float* lsp = nullptr;
      if (kLseLike || KIND == kEpiGrad) {
        bool live = rv;
        if (KIND == kEpiGrad) {
          cn = (rv && ep.rowmask[grow]) ? g_scale : 0.f;
          live = (cn != 0.f);
          if (live) {
            lse_l2 = ep.lse[grow] * kLog2e;
            cnw = cn * ep.wsum[grow];
          }
        }
        if (live) {
          lst = ep.sidx + grow * ep.Kp;
          lsp = ep.sprob + grow * ep.Kp;
          kpos = lower_bound_list(lst, ep.Kp, t0 * BN);
          if (!dbg_ok(kpos < ep.Kp, ep.flags)) kpos = ep.Kp - 1;
          nxt = lst[kpos];
          nxtp = lsp[kpos];
        }
      }
      for (int t = t0; t < t1; ++t) {
        const long long c0 = rc.now();
        const bool got_acc = mbar_wait(&acc_full[acc], acc_phase, ab);
        rc.wait0(c0);
        rc.count();
        if (!got_acc) goto epi_done;
        tc_fence_after();
        const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(acc * C::kAccStride);
        // columns of this tile: [t * BN, col_lim); a last 32-column chunk that runs past
        // BN reads unused TMEM columns, which the stores below skip
        const int col_lim = min(ep.Ncols, t * BN + BN);
        // dW: a 32-column chunk that lies inside the tile goes through TMA (columns past d
        // and rows past V are clipped by the tensor map); with BN = 240 the last chunk holds
        // 16 columns and takes the per-thread path.  When accumulating, the old block of
        // chunk c + 1 is loaded while chunk c is processed.
        auto dw_tma_chunk = [&](int cc) {
          const int cl = t * BN + cc * 32;
          return cl < col_lim && cl + 32 <= t * BN + BN;
        };
        auto dw_load = [&](int cc, int b) {
          if (lane == 0) {
            bulk_wait_read<0>();   // the last store out of buffer b has read it
            mbar_arrive_expect_tx(&wbar[b], 4096);
            const int lx = t * BN + cc * 32;
            tma_load_2d(wbuf + b * 4096, &tmOut, &wbar[b], dbg_ok((lx & 3) == 0, ep.flags) ? lx : (lx & ~3),
                        row0 + q * 32);
          }
          dw_pending |= 1u << b;
          __syncwarp();
        };
        if (KIND == kEpiRmwF32 && ep.accumulate && dw_tma_chunk(0)) dw_load(0, sbuf);
#pragma unroll 1
        for (int c = 0; c < (BN + 31) / 32; ++c) {
          const int col = t * BN + c * 32;
          if (col >= col_lim) break;
          if (KIND == kEpiRmwF32 && ep.accumulate && dw_tma_chunk(c) && dw_tma_chunk(c + 1))
            dw_load(c + 1, sbuf ^ 1);
          float v[32];
          tmem_ld32(tbase + c * 32, v);
          tmem_wait_ld();
          if (kLseLike) {
            if (KIND == kEpiLseStore) {
              // stage the warp's 32 rows x 32 fp32 logits (128-byte swizzle: 16-byte
              // chunk q of row r at chunk q ^ (r & 7)) and store them with TMA; columns
              // past V and rows past the chunk are clipped by the tensor map
              uint8_t* buf = wbuf + sbuf * 4096;
              if (lane == 0) bulk_wait_read<1>();
              __syncwarp();
              const uint32_t sw = static_cast<uint32_t>(lane & 7);
              const uint32_t row_addr = smem_u32(buf) + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
              for (int c16 = 0; c16 < 8; ++c16)
                st_shared_v4(row_addr + ((static_cast<uint32_t>(c16) ^ sw) << 4), __float_as_uint(v[c16 * 4 + 0]),
                             __float_as_uint(v[c16 * 4 + 1]), __float_as_uint(v[c16 * 4 + 2]),
                             __float_as_uint(v[c16 * 4 + 3]));
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0 && dbg_ok((col & 3) == 0 && col >= 0 && row0 + q * 32 >= 0, ep.flags)) {
                tma_store_2d(&tmOut, buf, col, row0 + q * 32);
                bulk_commit();
              }
              sbuf ^= 1;
            }
            if (col + 32 > ep.Ncols) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col + j >= ep.Ncols) v[j] = -INFINITY;
            }
            float cm = v[0];
#pragma unroll
            for (int j = 1; j < 32; ++j) cm = fmaxf(cm, v[j]);
            const float mn = fmaxf(m_run, cm);
            const float ms = mn * es;
            float acc_s = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) acc_s += ex2_approx(fmaf(v[j], es, -ms));
            s_run = s_run * ex2_approx((m_run - mn) * es) + acc_s;
            m_run = mn;
            while (nxt < col + 32) {
              if (!dbg_ok(nxt >= col && kpos + 1 < ep.Kp, ep.flags)) {
                nxt = kSentinel;
                break;
              }
              a_run = fmaf(nxtp, pick32(v, static_cast<uint32_t>(nxt - col)), a_run);
              ++kpos;
              nxt = lst[kpos];
              nxtp = lsp[kpos];
            }
          } else if (KIND == kEpiGrad) {
            float g[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) g[j] = cnw * ex2_approx(fmaf(v[j], es, -lse_l2));
            while (nxt < col + 32) {
              if (!dbg_ok(nxt >= col && kpos + 1 < ep.Kp, ep.flags)) {
                nxt = kSentinel;
                break;
              }
              const uint32_t off = static_cast<uint32_t>(nxt - col);
              const float cp = cn * nxtp;
#pragma unroll
              for (int j = 0; j < 32; ++j) g[j] = (off == static_cast<uint32_t>(j)) ? g[j] - cp : g[j];
              ++kpos;
              nxt = lst[kpos];
              nxtp = lsp[kpos];
            }
            // stage 32 rows x 32 columns (bf16, 64-byte swizzle) and store with TMA
            uint8_t* buf = wbuf + sbuf * 2048;
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
            const uint32_t row_addr = smem_u32(buf) + static_cast<uint32_t>(lane) * 64u;
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16)
              st_shared_v4(row_addr + ((static_cast<uint32_t>(c16) ^ sw) << 4),
                           pack_bf16x2(g[c16 * 8 + 0], g[c16 * 8 + 1]), pack_bf16x2(g[c16 * 8 + 2], g[c16 * 8 + 3]),
                           pack_bf16x2(g[c16 * 8 + 4], g[c16 * 8 + 5]), pack_bf16x2(g[c16 * 8 + 6], g[c16 * 8 + 7]));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && dbg_ok((col & 7) == 0 && col >= 0 && row0 + q * 32 >= 0, ep.flags)) {
              tma_store_2d(&tmOut, buf, col, row0 + q * 32);
              bulk_commit();
            }
            sbuf ^= 1;
          } else if (KIND == kEpiStoreBf16) {
            if (rv) {
              uint16_t* dst = ep.dH + grow * ep.ldo + col;
#pragma unroll
              for (int g8 = 0; g8 < 4; ++g8) {
                if (col + g8 * 8 + 8 <= col_lim) {
                  uint4 pk;
                  pk.x = pack_bf16x2(v[g8 * 8 + 0], v[g8 * 8 + 1]);
                  pk.y = pack_bf16x2(v[g8 * 8 + 2], v[g8 * 8 + 3]);
                  pk.z = pack_bf16x2(v[g8 * 8 + 4], v[g8 * 8 + 5]);
                  pk.w = pack_bf16x2(v[g8 * 8 + 6], v[g8 * 8 + 7]);
                  *reinterpret_cast<uint4*>(dst + g8 * 8) = pk;
                }
              }
            }
          } else if (KIND == kEpiTopK) {
            const int Kh = ep.topk_K;
            // candidates above the current root (a stale root only admits extras,
            // which the exact test below rejects), taken in column order
            uint32_t cand = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) cand |= (v[j] > hroot) ? (1u << j) : 0u;
            if (col + 32 > ep.Ncols) cand &= (1u << (ep.Ncols - col)) - 1u;
            while (cand) {
              const int j = __ffs(cand) - 1;
              cand &= cand - 1u;
              const float val = pick32(v, static_cast<uint32_t>(j));
              const int vi = col + j - ubase;
              if (hcnt < Kh) {
                // still filling: append and sift up.  Within a unit columns arrive in
                // increasing order, so a later column of equal value ranks lower.
                int pos = hcnt++;
                while (pos > 0) {
                  const int par = (pos - 1) >> 1;
                  const float pv = hv[par * kBM];
                  const int pi = hi[par * kBM];
                  if (pv < val || (pv == val && pi > vi)) break;   // the parent ranks lower
                  hv[pos * kBM] = pv;
                  hi[pos * kBM] = static_cast<uint16_t>(pi);
                  pos = par;
                }
                hv[pos * kBM] = val;
                hi[pos * kBM] = static_cast<uint16_t>(vi);
                if (hcnt == Kh) hroot = hv[0];
              } else if (val > hroot) {
                // replace the root (the smallest kept entry) and sift down; ties keep the
                // earlier index
                int pos = 0;
                while (true) {
                  const int l = 2 * pos + 1;
                  if (l >= Kh) break;
                  int c = l;
                  float cv = hv[l * kBM];
                  int ci = hi[l * kBM];
                  if (l + 1 < Kh) {
                    const float rv2 = hv[(l + 1) * kBM];
                    const int ri2 = hi[(l + 1) * kBM];
                    if (rv2 < cv || (rv2 == cv && ri2 > ci)) {
                      c = l + 1;
                      cv = rv2;
                      ci = ri2;
                    }
                  }
                  if (cv > val || (cv == val && ci < vi)) break;   // child ranks above the new entry
                  hv[pos * kBM] = cv;
                  hi[pos * kBM] = static_cast<uint16_t>(ci);
                  pos = c;
                }
                hv[pos * kBM] = val;
                hi[pos * kBM] = static_cast<uint16_t>(vi);
                hroot = hv[0];
              }
            }
          } else {  // kEpiRmwF32
            const int wrow0 = row0 + q * 32;
            if (dw_tma_chunk(c)) {
              // the warp's 32 rows x 32 fp32 columns in the 128-byte-swizzled layout of the
              // tensor map (16-byte chunk c16 of row r at c16 ^ (r & 7)): thread = row
              uint8_t* buf = wbuf + sbuf * 4096;
              const uint32_t sw = static_cast<uint32_t>(lane & 7);
              const uint32_t row_addr = smem_u32(buf) + static_cast<uint32_t>(lane) * 128u;
              if (ep.accumulate) {
                if (!mbar_wait(&wbar[sbuf], (dw_phase >> sbuf) & 1u, ab)) goto epi_done;
                dw_phase ^= 1u << sbuf;
                dw_pending &= ~(1u << sbuf);
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                  const float4 o = ld_shared_v4f(row_addr + ((static_cast<uint32_t>(c16) ^ sw) << 4));
                  v[c16 * 4 + 0] += o.x;
                  v[c16 * 4 + 1] += o.y;
                  v[c16 * 4 + 2] += o.z;
                  v[c16 * 4 + 3] += o.w;
                }
              } else {
                if (lane == 0) bulk_wait_read<1>();   // the store before last out of this buffer has read it
                __syncwarp();
              }
#pragma unroll
              for (int c16 = 0; c16 < 8; ++c16)
                st_shared_v4(row_addr + ((static_cast<uint32_t>(c16) ^ sw) << 4), __float_as_uint(v[c16 * 4 + 0]),
                             __float_as_uint(v[c16 * 4 + 1]), __float_as_uint(v[c16 * 4 + 2]),
                             __float_as_uint(v[c16 * 4 + 3]));
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0 && dbg_ok((col & 3) == 0 && col >= 0 && wrow0 >= 0, ep.flags)) {
                tma_store_2d(&tmOut, buf, col, wrow0);
                bulk_commit();
              }
              sbuf ^= 1;
            } else if (rv) {
              // a chunk cut by the tile edge: this thread's own row, element by element
              float* dst = ep.dW + static_cast<int64_t>(row) * ep.ldo;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col + j < col_lim) dst[col + j] = (ep.accumulate ? dst[col + j] : 0.f) + v[j];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_cluster(acc_empty0 + static_cast<uint32_t>(acc) * 8u);
          else mbar_arrive(&acc_empty[acc]);
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (KIND == kEpiTopK && rv) {
        const int64_t slot = (uslot * C::kMmaM + static_cast<int>(rank) * kBM + row_local) *
                             ep.topk_K;
        const int kw = dbg_ok(slot + ep.topk_K <= ep.topk_cap, ep.flags) ? ep.topk_K : 0;
        for (int k = 0; k < kw; ++k) {
          const int rel = hi[k * kBM];
          ep.part_tv[slot + k] = hv[k * kBM];
          ep.part_ti[slot + k] = rel == kTopKEmpty ? kSentinel : ubase + rel;
        }
      }
      if (kLseLike && rv) {
        const int64_t slot = uslot * C::kMmaM + static_cast<int>(rank) * kBM + row_local;
        if (dbg_ok(slot < ep.part_cap, ep.flags)) {
          ep.part_m[slot] = m_run;
          ep.part_s[slot] = s_run;
          ep.part_a[slot] = a_run;
        }
      }
    }
  epi_done:
    if (q == 0 && lane == 0) rc.flush(KIND, 8);
    if (KIND == kEpiRmwF32 && lane == 0 && dw_pending) {
      // a load of an old dW block may still be landing (abort path): bounded wait
      const uint64_t w0 = globaltimer_ns();
      for (int b2 = 0; b2 < 2; ++b2)
        if (dw_pending & (1u << b2))
          while (!mbar_try_wait(smem_u32(&wbar[b2]), (dw_phase >> b2) & 1u) && globaltimer_ns() - w0 < kDrainLimitNs) {
          }
    }
    if (KIND == kEpiGrad || KIND == kEpiLseStore || KIND == kEpiRmwF32) {
      if (lane == 0) bulk_wait<0>();
      __syncwarp();
    }
  }

  if (*abort_flag) {
    // give copies that may still be landing in shared memory time to finish
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 1000000ull) {
    }
  }
  tc_fence_before();
  if (PAIR) cluster_sync();   // the peer's shared memory and TMEM stay alive until the pair is done
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int KIND, int BN, bool PAIR>
static cudaError_t launch_one(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmOut,
                              const Sched& sc, const EpiParams& ep, int grid, cudaStream_t stream) {
  using C = GemmCfg<KIND, BN, PAIR>;
  // the dynamic shared-memory limit is a per-device attribute: set it on the first
  // launch on each device (devices past the 64th get it on every launch)
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit == 0 || !(configured.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(gemm_kernel<KIND, BN, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  if (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(192, 1, 1);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_kernel<KIND, BN, PAIR>, tmA, tmB, tmOut, sc, ep);
  }
  gemm_kernel<KIND, BN, PAIR><<<grid, 192, C::kSmem, stream>>>(tmA, tmB, tmOut, sc, ep);
  return cudaGetLastError();
}

cudaError_t launch_gemm(int kind, int BN, bool pair, const CUtensorMap& tmA, const CUtensorMap& tmB,
                        const CUtensorMap& tmOut, const Sched& sc, const EpiParams& ep, int grid,
                        cudaStream_t stream) {
  if (pair) {
    // the loss and top-K GEMMs always use 256-wide tiles; dHidden / dW any pair width
#define KDKL_PAIR_WIDTHS(KIND_)                                                                   \
  switch (BN) {                                                                                   \
    case 256: return launch_one<KIND_, 256, true>(tmA, tmB, tmOut, sc, ep, grid, stream);        \
    case 240: return launch_one<KIND_, 240, true>(tmA, tmB, tmOut, sc, ep, grid, stream);        \
    case 224: return launch_one<KIND_, 224, true>(tmA, tmB, tmOut, sc, ep, grid, stream);        \
    case 192: return launch_one<KIND_, 192, true>(tmA, tmB, tmOut, sc, ep, grid, stream);        \
    case 160: return launch_one<KIND_, 160, true>(tmA, tmB, tmOut, sc, ep, grid, stream);        \
    case 128: return launch_one<KIND_, 128, true>(tmA, tmB, tmOut, sc, ep, grid, stream);        \
    default: return cudaErrorInvalidValue;                                                        \
  }
    switch (kind) {
      case kEpiLse:
        if (BN != 256) return cudaErrorInvalidValue;
        return launch_one<kEpiLse, 256, true>(tmA, tmB, tmOut, sc, ep, grid, stream);
      case kEpiLseStore:
        if (BN != 256) return cudaErrorInvalidValue;
        return launch_one<kEpiLseStore, 256, true>(tmA, tmB, tmOut, sc, ep, grid, stream);
      case kEpiGrad:
        if (BN != 256) return cudaErrorInvalidValue;
        return launch_one<kEpiGrad, 256, true>(tmA, tmB, tmOut, sc, ep, grid, stream);
      case kEpiTopK:
        if (BN != 256) return cudaErrorInvalidValue;
        return launch_one<kEpiTopK, 256, true>(tmA, tmB, tmOut, sc, ep, grid, stream);
      case kEpiStoreBf16: KDKL_PAIR_WIDTHS(kEpiStoreBf16)
      case kEpiRmwF32: KDKL_PAIR_WIDTHS(kEpiRmwF32)
      default: return cudaErrorInvalidValue;
    }
#undef KDKL_PAIR_WIDTHS
  }
  switch (kind) {
    case kEpiLse:
      return launch_one<kEpiLse, 256, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
    case kEpiLseStore:
      return launch_one<kEpiLseStore, 256, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
    case kEpiGrad:
      return launch_one<kEpiGrad, 256, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
    case kEpiStoreBf16:
      if (BN == 256) return launch_one<kEpiStoreBf16, 256, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
      if (BN == 192) return launch_one<kEpiStoreBf16, 192, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
      if (BN == 128) return launch_one<kEpiStoreBf16, 128, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
      break;
    case kEpiRmwF32:
      if (BN == 256) return launch_one<kEpiRmwF32, 256, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
      if (BN == 192) return launch_one<kEpiRmwF32, 192, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
      if (BN == 128) return launch_one<kEpiRmwF32, 128, false>(tmA, tmB, tmOut, sc, ep, grid, stream);
      break;
    default:
      break;
  }
  return cudaErrorInvalidValue;
}

// ============================================================================
// self-test of the bounded wait: one thread waits on an mbarrier that nothing
// completes; the wait must give up after `limit_ns`, set the timeout bit of the
// flag word and let the kernel return normally (the context stays usable).
// ============================================================================
__global__ void wait_selftest_kernel(uint32_t* flags, uint64_t limit_ns, uint64_t* waited_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  fence_mbar_init();
  AbortState ab{&abort_flag, flags};
  ab.limit_ns = limit_ns;
  const uint64_t t0 = globaltimer_ns();
  const bool ok = mbar_wait(&bar, 0, ab);
  *waited_ns = globaltimer_ns() - t0;
  if (ok) atomicOr(flags, 0x80000000u);   // cannot happen: nothing arrives on the barrier
}

cudaError_t launch_wait_selftest(uint32_t* flags, uint64_t limit_ns, uint64_t* waited_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(flags, limit_ns, waited_ns);
  return cudaGetLastError();
}

// ============================================================================
// G from stored logits (fused forward + backward).  For each row n of a chunk:
//   G[n, v] = c_n (w_n 2^{z[n, v] log2e / tau_s - lse_n log2e} - target[n, v])  (bf16),
// c_n = m_n g / (tau_s N_valid), with the gradient epilogue's instructions in the
// same order, so that for the same z and lse the result is the same bits.  One
// block per row; warp w covers the 128-column groups w, w + 8, ... (lane l holds
// 4 columns), and the row's sorted target list is walked forward once per warp.
// ============================================================================
constexpr int kGPassThreads = 256;

__global__ void __launch_bounds__(kGPassThreads)
    gpass_kernel(const float* __restrict__ z, int64_t ldz, uint16_t* __restrict__ G, int64_t ldg, int V,
                 int64_t row_offset, const int* __restrict__ sidx, const float* __restrict__ sprob, int Kp,
                 const uint8_t* __restrict__ rowmask, const float* __restrict__ wsum,
                 const float* __restrict__ lse, const uint32_t* __restrict__ n_valid,
                 const float* __restrict__ grad_loss, float inv_tau_s, float exp_scale, uint32_t* __restrict__ flags) {
  const int64_t n = blockIdx.x;
  const int64_t grow = row_offset + n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t nv = *n_valid;
  const float g = grad_loss ? *grad_loss : 1.0f;
  const float g_scale = nv > 0 ? g * inv_tau_s / static_cast<float>(nv) : 0.f;
  const float cn = rowmask[grow] ? g_scale : 0.f;
  uint16_t* grow_out = G + n * ldg;
  const float* zrow = z + n * ldz;
  const int groups = (V + 127) / 128;
  if (cn == 0.f) {
    for (int gi = warp; gi < groups; gi += kGPassThreads / 32) {
      const int c0 = gi * 128 + lane * 4;
      if (c0 + 3 < V) {
        *reinterpret_cast<uint2*>(grow_out + c0) = make_uint2(0u, 0u);
      } else {
        for (int j = 0; j < 4; ++j)
          if (c0 + j < V) grow_out[c0 + j] = 0;
      }
    }
    return;
  }
  const float es = exp_scale;
  const float lse_l2 = lse[grow] * kLog2e;
  const float cnw = cn * wsum[grow];
  const int* lst = sidx + grow * Kp;
  const float* lsp = sprob + grow * Kp;
  // four 128-column groups per pass: their loads are all in flight before any is used
  constexpr int kStride = kGPassThreads / 32;
  constexpr int kU = 4;
  int kpos = lower_bound_list(lst, Kp, warp * 128);
  for (int gb = warp; gb < groups; gb += kStride * kU) {
    float v[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c0 = (gb + u * kStride) * 128 + lane * 4;
      if (c0 + 3 < V) {
        const float4 q = *reinterpret_cast<const float4*>(zrow + c0);
        v[u][0] = q.x;
        v[u][1] = q.y;
        v[u][2] = q.z;
        v[u][3] = q.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[u][j] = (c0 + j < V) ? zrow[c0 + j] : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int gi = gb + u * kStride;
      if (gi >= groups) break;
      const int g0 = gi * 128;
      const int c0 = g0 + lane * 4;
      float gv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) gv[j] = cnw * ex2_approx(fmaf(v[u][j], es, -lse_l2));
      while (lst[kpos] < g0 && dbg_ok(kpos + 1 < Kp, flags)) ++kpos;
      for (int k = kpos; lst[k] < g0 + 128 && dbg_ok(k + 1 < Kp, flags); ++k) {
        const uint32_t off = static_cast<uint32_t>(lst[k] - c0);
        const float cp = cn * lsp[k];
#pragma unroll
        for (int j = 0; j < 4; ++j) gv[j] = (off == static_cast<uint32_t>(j)) ? gv[j] - cp : gv[j];
      }
      if (c0 + 3 < V) {
        *reinterpret_cast<uint2*>(grow_out + c0) =
            make_uint2(pack_bf16x2(gv[0], gv[1]), pack_bf16x2(gv[2], gv[3]));
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (c0 + j < V) grow_out[c0 + j] = static_cast<uint16_t>(pack_bf16x2(gv[j], 0.f) & 0xFFFFu);
      }
    }
  }
}

cudaError_t launch_gpass(const float* z, int64_t ldz, uint16_t* G, int64_t ldg, int64_t nc, int V,
                         int64_t row_offset, const int* sidx, const float* sprob, int Kp, const uint8_t* rowmask,
                         const float* wsum, const float* lse, const uint32_t* n_valid, const float* grad_loss,
                         float student_tau, uint32_t* flags, cudaStream_t stream) {
  if (nc <= 0) return cudaSuccess;
  gpass_kernel<<<static_cast<unsigned>(nc), kGPassThreads, 0, stream>>>(
      z, ldz, G, ldg, V, row_offset, sidx, sprob, Kp, rowmask, wsum, lse, n_valid, grad_loss, 1.0f / student_tau,
      1.4426950408889634f / student_tau, flags);
  return cudaGetLastError();
}

// ============================================================================
// top-K merge: one warp per row keeps the K best of the row's split heaps,
// ordered by value descending, then index ascending
// ============================================================================
constexpr int kMergeCand = kTopKMergeCand;   // splits * K never exceeds this (the planner caps splits)
constexpr int kTopKMergeWarps = 8;

// Orderable 64-bit key of a (logit, index) candidate: a larger key ranks
// earlier (larger logit, then smaller index).  -0 is folded into +0 so that
// equal logits tie on the index alone, as the comparison of values does.
__device__ __forceinline__ uint64_t topk_key(float v, int idx) {
  if (v == 0.0f) v = 0.0f;
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(u) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

__device__ __forceinline__ float topk_key_value(uint64_t key) {
  uint32_t u = static_cast<uint32_t>(key >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}

__device__ __forceinline__ int topk_key_index(uint64_t key) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}

// One warp per row: the row's S split heaps (S * K <= kMergeCand candidates,
// K <= kTopKMax) are reduced to the K best, best first.  The K-th largest key
// is found exactly by a radix select (one byte per pass, from the top, with a
// 256-bin warp histogram); the keys above it, plus as many copies of it as are
// still needed, are compacted with ballots and only those K are sorted.  The
// K best of V >= K columns are always real entries, so empty heap slots
// (-inf, sentinel index) never reach the output.
__global__ void __launch_bounds__(kTopKMergeWarps * 32)
    topk_merge_kernel(const float* __restrict__ part_tv, const int* __restrict__ part_ti, int splits,
                      int rows_per_block, int K, int64_t N, int32_t* __restrict__ topk_idx,
                      float* __restrict__ topk_logit, int64_t part_cap, uint32_t* __restrict__ flags) {
  constexpr int kPerLane = kMergeCand / 32;
  __shared__ uint32_t s_hist[kTopKMergeWarps][256];
  __shared__ uint64_t s_sel[kTopKMergeWarps][kTopKMax];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* hist = s_hist[w];
  uint64_t* sel = s_sel[w];
  const int C = splits * K;
  int P = 1;   // sort width of the K selected keys (a power of two <= kTopKMax)
  while (P < K) P <<= 1;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * kTopKMergeWarps + w; n < N;
       n += static_cast<int64_t>(gridDim.x) * kTopKMergeWarps) {
    const int64_t rb = n / rows_per_block;
    const int r = static_cast<int>(n - rb * rows_per_block);
    // candidate c = j * K + k (split j, heap slot k) sits in lane c % 32 as key[c / 32];
    // 0 ranks below every real key
    uint64_t key[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int c = lane + 32 * i;
      key[i] = 0;
      if (c < C) {
        const int j = c / K, k = c - j * K;
        const int64_t slot = ((rb * splits + j) * rows_per_block + r) * K + k;
        if (dbg_ok(slot < part_cap, flags)) key[i] = topk_key(part_tv[slot], part_ti[slot]);
      }
    }
    // radix select: after pass p, `prefix` holds the top p+1 bytes of the K-th
    // largest key and `need` counts the keys still to take among those sharing them
    uint64_t prefix = 0, pmask = 0;
    int need = K;
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int b = lane; b < 256; b += 32) hist[b] = 0;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if ((key[i] & pmask) == prefix) atomicAdd(&hist[(key[i] >> shift) & 0xFFu], 1u);
      __syncwarp();
      // lane l holds digits 255 - 8 l down to 248 - 8 l; lanes scan from the top
      uint32_t cnt[8];
      uint32_t tot = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        cnt[t] = hist[255 - 8 * lane - t];
        tot += cnt[t];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - tot;
      const bool here = excl < static_cast<uint32_t>(need) && incl >= static_cast<uint32_t>(need);
      const int src = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
      uint32_t digit = 0, above = excl;
      if (here) {
        bool found = false;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (!found) {
            if (above + cnt[t] >= static_cast<uint32_t>(need)) {
              digit = static_cast<uint32_t>(255 - 8 * lane - t);
              found = true;
            } else {
              above += cnt[t];
            }
          }
        }
      }
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      need -= static_cast<int>(above);
      prefix |= static_cast<uint64_t>(digit) << shift;
      pmask |= 0xFFull << shift;
      __syncwarp();
    }
    // keep the keys above the K-th, then `need` copies of it
    const uint64_t kth = prefix;
    int base = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const bool take = key[i] > kth;
      const uint32_t b = __ballot_sync(0xffffffffu, take);
      if (take && dbg_ok(base + __popc(b & ((1u << lane) - 1u)) < kTopKMax, flags))
        sel[base + __popc(b & ((1u << lane) - 1u))] = key[i];
      base += __popc(b);
    }
    for (int k = base + lane; k < K; k += 32) sel[k] = kth;
    for (int k = K + lane; k < P; k += 32) sel[k] = 0;
    __syncwarp();
    // bitonic sort of the P selected keys, largest first
    for (int k2 = 2; k2 <= P; k2 <<= 1) {
      for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
        for (int i = lane; i < P; i += 32) {
          const int l = i ^ j2;
          if (l > i) {
            const uint64_t a = sel[i], b = sel[l];
            const bool first_block = (i & k2) == 0;
            if (first_block ? (a < b) : (a > b)) {
              sel[i] = b;
              sel[l] = a;
            }
          }
        }
        __syncwarp();
      }
    }
    for (int k = lane; k < K; k += 32) {
      const uint64_t kk = sel[k];
      topk_logit[n * K + k] = topk_key_value(kk);
      topk_idx[n * K + k] = topk_key_index(kk);
    }
    __syncwarp();
  }
}

cudaError_t launch_topk_merge(const float* part_tv, const int* part_ti, int splits, int rows_per_block, int K,
                              int64_t N, int32_t* topk_idx, float* topk_logit, int64_t part_cap, uint32_t* flags,
                              cudaStream_t stream) {
  if (splits * K > kMergeCand) return cudaErrorInvalidValue;
  const int64_t blocks = (N + kTopKMergeWarps - 1) / kTopKMergeWarps;
  const int grid = static_cast<int>(blocks < 4096 ? blocks : 4096);
  topk_merge_kernel<<<grid, kTopKMergeWarps * 32, 0, stream>>>(part_tv, part_ti, splits, rows_per_block, K, N,
                                                                topk_idx, topk_logit, part_cap, flags);
  return cudaGetLastError();
}

}  // namespace kdkl

#if defined(KDKL_PROFILE)
// Host side of the role cycle counters (declared in kdkl_profile.h).
#include "../../include/kdkl_profile.h"

extern "C" kdkl_status kdkl_profile_role_cycles_shape(int32_t* kinds, int32_t* ctas, int32_t* slots) {
  if (!kinds || !ctas || !slots) return KDKL_ERR_NULL;
  *kinds = kdkl::kRoleKinds;
  *ctas = kdkl::kRoleCtas;
  *slots = kdkl::kRoleSlots;
  return KDKL_OK;
}

extern "C" kdkl_status kdkl_profile_read_role_cycles(void* host_dst, size_t bytes) {
  if (!host_dst) return KDKL_ERR_NULL;
  if (bytes != sizeof(kdkl::g_role_cycles)) return KDKL_ERR_SHAPE;
  return cudaMemcpyFromSymbol(host_dst, kdkl::g_role_cycles, bytes) == cudaSuccess ? KDKL_OK : KDKL_ERR_CUDA;
}

extern "C" kdkl_status kdkl_profile_clear_role_cycles(void* stream) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, kdkl::g_role_cycles) != cudaSuccess) return KDKL_ERR_CUDA;
  return cudaMemsetAsync(p, 0, sizeof(kdkl::g_role_cycles), static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDKL_OK
             : KDKL_ERR_CUDA;
}
#endif
