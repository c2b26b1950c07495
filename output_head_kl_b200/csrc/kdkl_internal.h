// Internal declarations shared by the host API and the kernels (not installed).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace kdkl {

constexpr int kBM = 128;        // rows of one MMA tile (TMEM lanes)
constexpr int kBK = 64;         // K elements per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kMaxK = 256;      // cached entries per row
constexpr int kSentinel = 0x7FFFFFFF;  // pads each row's sorted index list

// Row-pitch (in int32/f32 elements) of the per-row sorted target list:
// room for the K cached entries and a hard label, then at least one sentinel,
// rounded to 4.
inline int list_pitch(int K) { return ((K + 2) + 3) & ~3; }   // K entries + a hard label + a sentinel

// Workspace layout (all offsets 256-byte aligned).  Header words:
//   [0] device flag word (KDKL_DEV_* bits)
//   [1] N_valid (count of rows that enter the loss)
//   [2] ticket of the loss reduction
struct WsLayout {
  size_t header = 0;       // 256 bytes
  size_t sync = 0;         // [kSyncSlots] uint64 positions of a synchronised GEMM launch
  size_t sidx = 0;         // [N, Kp] int32 sorted unique indices (sentinel padded)
  size_t sprob = 0;        // [N, Kp] f32 teacher probabilities aligned with sidx
  size_t negent = 0;       // [N] f32 gamma * sum_v P_T log P_T of the teacher row
  size_t wsum = 0;         // [N] f32 total target weight of the row (gamma + beta if it has a label)
  size_t rowmask = 0;      // [N] uint8 effective mask (mask and row usable)
  size_t partial = 0;      // [units_cap * 128] x 3 f32 (running max, sum-exp, gathered logit)
  size_t blocksum = 0;     // [ceil(N / 256)] f64 loss partial sums
  size_t gbuf = 0;         // [chunk, Vp] bf16 chunk buffer of the logit gradient
  size_t total = 0;
  int Kp = 0;
  int64_t units_cap = 0;
  int64_t chunk = 0;
  int64_t Vp = 0;
};

WsLayout make_layout(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens);

// Work decomposition shared by every role of a GEMM kernel.
//   row-stream mode: unit u -> row block u / splits, vocabulary tiles
//     [(j * n_tiles) / splits, ((j + 1) * n_tiles) / splits) with j = u % splits.
//   tile mode: unit u -> row block u / n_tiles, the single tile u % n_tiles.
// Work units of a persistent GEMM launch, dealt round-robin to the CTA groups.
//   row_stream = 0: one output tile per unit, u = row block * n_tiles + tile, or with
//     col_group > 0 the tiles in groups of col_group columns, each group swept row
//     block by row block (fewer B columns in flight at once, more passes over A);
//   row_stream = kRowMajor: a unit is (row block, vocabulary split) and sweeps the
//     split's tiles, u = row block * splits + split (the row blocks in flight stay few);
//   row_stream = kSplitMajor: the same units, dealt in groups of rb_group row blocks
//     (0 = all of them): within a group u = split * rows of the group + row block, so
//     the CTA groups running at once cover every row block of the group for one split
//     and share its W tiles, while only the group's hidden rows need to stay in L2.
constexpr int kRowMajor = 1;
constexpr int kSplitMajor = 2;
//
// Lockstep of a row-stream launch (sync_window > 0): the CTA groups that run units of
// the same vocabulary split in the same round (round k = units [k G, k G + G) for G
// groups; group g runs unit g + k G) stream the same W tiles, which only one DRAM
// read serves while they stay close together.  Each group publishes its position
// (unit + 1) << 32 | (tile - first tile of the unit) in prog[group] as it reaches a
// tile, and the even CTA's producer then holds back tile r of a unit until every peer
// group of that round and split has reached tile r - sync_window.  Tile-mode launches
// (dHidden, dW: one long reduction per unit, and the units of a round share rows of A
// or columns of B) do the same every kSyncKStep reduction blocks, with every unit of
// the round as a peer and sync_window counted in reduction blocks.  prog must be
// zeroed before the launch.  A wait that lasts longer than kSyncSoftLimitNs gives
// up and the group stops holding back for the rest of its unit; waiting never
// changes results, only how far the groups drift apart.
enum L2Priority { kL2Normal = 0, kL2Last = 1, kL2First = 2 };
constexpr int kSyncSlots = 1024;                          // groups a synchronised launch may have
constexpr int kSyncKStep = 16;                            // tile mode: reduction blocks per position step
constexpr unsigned long long kSyncSoftLimitNs = 1000000;  // 1 ms
struct Sched {
  int units;
  int splits;
  int n_tiles;
  int k_blocks;
  int row_stream;
  int sync_window;
  unsigned long long* prog;
  // L2 eviction priority of the A and B operand loads (kL2Normal = 0, kL2Last, kL2First)
  int l2_a;
  int l2_b;
  int rb_group;   // kSplitMajor: row blocks per group (0 = all)
  int col_group;  // tile mode: column tiles per group (0 = all; u = row block * n_tiles + tile)
  int die_order;  // number the CTA groups by the half of the SM ids they run on (prog[ngroups..+1] = tickets)
};

// Parameters of the fused epilogues (the union of what each kind needs).
struct EpiParams {
  // geometry
  int M;             // valid rows of the A operand (tokens of the chunk, or V for dW)
  int Ncols;         // valid columns of the output (V for loss tiles, d for gradients)
  int64_t row_offset;  // global token index of local row 0
  // teacher lists and per-row data (indexed by global token)
  const int* sidx;
  const float* sprob;
  int Kp;
  const uint8_t* rowmask;
  // forward partials (part_cap slots per plane)
  float* part_m;
  float* part_s;
  float* part_a;
  int64_t part_cap;
  // student temperature: exp_scale = log2(e) / tau_s, inv_tau_s = 1 / tau_s
  float exp_scale;
  float inv_tau_s;
  const float* wsum;           // per-row total target weight
  // backward scale
  const float* lse;
  const float* grad_loss;      // may be null (1.0)
  const uint32_t* n_valid;     // device counter
  // gradient outputs
  uint16_t* dH;        // bf16 bits [N, d]
  float* dW;           // [V, d]
  int ldo;             // row pitch (elements) of dH / dW
  int accumulate;      // dW: add into the existing values
  uint32_t* flags;     // device flag word
  // teacher top-K producer: K per row, partial heaps [units * rows_per_unit, K]
  int topk_K;
  float* part_tv;
  int* part_ti;
  int64_t topk_cap;    // entries of part_tv / part_ti
};

// kEpiLseStore: the forward's online log-sum-exp and gather (as kEpiLse), and
// every fp32 logit tile also stored to a chunk buffer (fused forward + backward).
enum EpiKind { kEpiLse = 0, kEpiGrad = 1, kEpiStoreBf16 = 2, kEpiRmwF32 = 3, kEpiTopK = 4, kEpiLseStore = 5 };
// Shape of the profiling build's role cycle counters: [epilogue kind][CTA][slot].
constexpr int kRoleKinds = 8;
constexpr int kRoleCtas = 256;
constexpr int kRoleSlots = 12;

// Teacher top-K producer: per-row min-heaps of up to kTopKMax entries live in
// shared memory during the vocabulary sweep, with 16-bit indices relative to
// the unit's first column; a unit therefore spans at most kTopKUnitTiles
// 256-column tiles (the planner's vocabulary splits guarantee it), and
// kTopKEmpty (above every relative index) marks an empty heap slot.
constexpr int kTopKMax = 128;
constexpr int kTopKUnitTiles = 255;
constexpr int kTopKEmpty = 0xFFFF;
// Per-row candidates the top-K merge sorts (vocabulary splits x K).
constexpr int kTopKMergeCand = 1024;

// Launchers (defined in kernels.cu).  Each returns cudaGetLastError() of its launch.
// cache_format 0: int32 indices + fp32 logits; 1: uint16 indices + bf16 logits.
cudaError_t launch_prepass(int cache_format, const void* topk_idx, const void* topk_logit, const uint8_t* mask,
                           const int32_t* labels, int64_t N, int32_t V, int32_t K, float tau, float gamma,
                           float beta, int* sidx, float* sprob, float* negent, float* wsum, uint8_t* rowmask,
                           int Kp, uint32_t* header, cudaStream_t stream);

// G (bf16, row pitch ldg) from stored fp32 logits z (row pitch ldz) for the nc rows
// of a chunk starting at global row row_offset; see gpass_kernel.
cudaError_t launch_gpass(const float* z, int64_t ldz, uint16_t* G, int64_t ldg, int64_t nc, int V,
                         int64_t row_offset, const int* sidx, const float* sprob, int Kp, const uint8_t* rowmask,
                         const float* wsum, const float* lse, const uint32_t* n_valid, const float* grad_loss,
                         float student_tau, uint32_t* flags, cudaStream_t stream);

// launch_merge: rows [0, N) of the pointers given (a chunk passes offset per-row
// pointers); their 256-row block sums land at blocksum[block_base + b], and the
// launch that completes block total_blocks - 1 of the step (0 = this launch's
// grid) sums all total_blocks in order into *loss.  part_cap = slots per partial
// plane (checked in the bounds-checking build).
cudaError_t launch_merge(const float* part_m, const float* part_s, const float* part_a, int splits,
                         int rows_per_block, float student_tau, const float* negent, const float* wsum,
                         const uint8_t* rowmask, int64_t N, float* lse, float* loss, double* blocksum,
                         uint32_t* header, const uint32_t* n_valid, int64_t block_base, int64_t total_blocks,
                         int64_t part_cap, cudaStream_t stream);

// GEMM kinds: A/B majorness and epilogue are fixed per kind.
//   kEpiLse      : A = hidden K-major, B = W K-major, BN = 256, row-stream
//   kEpiGrad     : A = hidden K-major, B = W K-major, BN = 256, row-stream, TMA store of G
//   kEpiStoreBf16: A = G K-major,      B = W MN-major, BN from {256, 192, 128}, tile mode
//   kEpiRmwF32   : A = G MN-major,     B = hidden MN-major, BN from {256, 192, 128}, tile mode
// pair = true (BN = 256 only): clusters of two CTAs, 256-row tiles, each CTA
// loading its 128 rows of A and BN/2 rows of B (the B map's box must be BN/2
// rows for K-major B); grid must be even.  Units then cover 256 rows.
cudaError_t launch_gemm(int kind, int BN, bool pair, const CUtensorMap& tmA, const CUtensorMap& tmB,
                        const CUtensorMap& tmOut, const Sched& sched, const EpiParams& ep, int grid,
                        cudaStream_t stream);

// Merges the per-split heaps of the top-K producer into each row's K entries,
// ordered by (logit descending, index ascending).
cudaError_t launch_topk_merge(const float* part_tv, const int* part_ti, int splits, int rows_per_block, int K,
                              int64_t N, int32_t* topk_idx, float* topk_logit, int64_t part_cap, uint32_t* flags,
                              cudaStream_t stream);

// Bounded-wait self-test (see kdkl_selftest_wait_timeout).
cudaError_t launch_wait_selftest(uint32_t* flags, uint64_t limit_ns, uint64_t* waited_ns, cudaStream_t stream);

// Sets the message kdkl_last_error() returns on this host thread.
void set_last_error(const char* msg);

}  // namespace kdkl
