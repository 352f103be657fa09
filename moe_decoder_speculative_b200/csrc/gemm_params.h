// Parameters of the grouped tensor-core GEMM engine (gemm_tc.cu).
#pragma once

#include <cstdint>
#include <cuda.h>

namespace mv {

enum { EPI_SWIGLU = 0, EPI_STORE_F32 = 1, EPI_ARGMAX = 2, EPI_SWIGLU_ROWS = 3, EPI_STORE_ROWS = 4, EPI_TOPK = 5,
       EPI_STORE_BF16 = 6,    // bf16(res + acc), res nullable (swap-AB tiles)
       EPI_ARGMAX_ROWS = 7 }; // CTA pairs, tokens on M: one argmax key per (token, 256 vocabulary rows)
// Operand modes.  The first four put weights on the MMA's M side (swap-AB);
// the tokens-on-M modes load the same tiles but multiply 128 token rows by 256
// weight rows (gate|up tiles, or two halves of W_down) into one accumulator.
enum { MODE_SINGLE = 0, MODE_GATEUP = 1, MODE_KPAIR = 2, MODE_MPAIR = 3, MODE_TGATEUP = 4, MODE_TPAIR = 5,
       MODE_TROUTE = 6,  // 128 token rows x the M (<= 256) router rows, one accumulator
       MODE_TLM = 7 };   // CTA pairs: 256 token rows x 256 LM-head rows (128 of each per CTA)
enum { GEMM_MOE_DECODE = 0, GEMM_MOE_PREFILL = 1, GEMM_LM = 2, GEMM_LM_WIDE = 3, GEMM_MOE_DECODE_FEW = 4 };

// B-operand TMA box height (rows) of each tile configuration; the host builds
// the B tensor maps with it.  Whole 128-row token tiles in one box matter: on
// the 9,248-row prefill layer 128-row boxes ran the grouped GEMM in 616 us
// against 757 us with 16-row boxes (8 boxes per stage).
#ifndef MV_PREFILL_BBOX
#define MV_PREFILL_BBOX 128
#endif
constexpr int kDecodeBBox = 32;  // GEMM_MOE_DECODE: one 3D box of 32 token rows x two k-blocks
constexpr int kPrefillBBox = MV_PREFILL_BBOX;
constexpr int kLmBBox = 16;       // GEMM_LM: few token rows
// CTA-pair prefill GEMM: 64-wide k-blocks per stage (1: 2D boxes, six 32 KB
// stages; 2: 3D boxes, three 64 KB stages).
#ifndef MV_PAIR_KB
#define MV_PAIR_KB 2
#endif
constexpr int kPairKB = MV_PAIR_KB;
constexpr int kLmWideBBox = 128;  // GEMM_LM_WIDE: 128 or more token rows

// Sticky device error bits, OR-ed into the workspace's error word.
constexpr int kErrTimeout = 1;
constexpr int kErrInternal = 2;

// Ints of scheduling state one grouped-GEMM launch uses (claim counter plus one
// completion counter per group); zeroed before the launch.
constexpr int kSchedInts = 1024;
constexpr int kMaxGroups = 2 * 256 + 8;  // routed + shared groups of both phases

// One operand set of the grouped GEMM: `groups` groups that share tensor maps.
// Group gi multiplies A rows [gi*a_group_stride, +M) by the B rows
// [offsets[gi], +counts[gi]) and writes output rows at the same B row index
// (EPI_SWIGLU: bf16 [rows][ld_out]; EPI_STORE_F32: fp32 [rows][ld_out];
// EPI_ARGMAX: uint64 keys [row][ld_out], one per (M tile, lane quarter)).
struct GemmSet {
  CUtensorMap a0;          // A operand
  CUtensorMap a1;          // second A operand (up weights), MODE_GATEUP only
  CUtensorMap b;           // B operand, box of 16 rows x 64 columns
  void* out;
  const int32_t* counts;   // device [groups] or nullptr (static_rows)
  const int32_t* offsets;  // device [groups], or nullptr: group g starts at row g * slab_rows
  int32_t slab_rows;       // rows reserved per group when offsets is nullptr (0: one group at row 0)
  int32_t ld_out;
  int32_t K;               // reduction length, multiple of 64
  int32_t M;               // valid A rows per group
  int32_t groups;
  int32_t static_rows;
  int32_t a_group_stride;
  int32_t mode;            // MODE_*
  int32_t epi;             // EPI_*
  int32_t m_tile;          // A rows per unit: 128, or 256 for MODE_MPAIR
  int32_t dep_set;         // -1, or the set whose same-index group must finish first
  int32_t signal;          // 1: count finished epilogue warps per group (a later set depends on it)
  int32_t key_row_base;    // EPI_ARGMAX: vocabulary index of this set's A row 0
  int32_t key_part_base;   // EPI_ARGMAX: first key slot of this set within a token's row
  void* out2;              // EPI_TOPK: fp32 weights [rows][topk] (`out` holds int32 ids [rows][topk])
  const float* bias;       // EPI_TOPK: fp32 [M] added to the logits, or nullptr
  int32_t topk;            // EPI_TOPK: k
  const uint16_t* res;     // EPI_STORE_BF16: bf16 [rows][ld_out] added before rounding, or nullptr
  const int32_t* row_map;  // EPI_STORE_F32 (swap-AB): output row of B row b is row_map[b], or nullptr: b
};

struct GemmParams {
  GemmSet set[4];
  int32_t nsets;
  int* err;
  int* sched;              // kSchedInts ints, zero at launch; nullptr: static round-robin units, no dependencies
  uint64_t timeout_ns;
};

}  // namespace mv
