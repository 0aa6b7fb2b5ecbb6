// Workspace layout and limits of the layer kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/pmoe.h"

namespace pmoe {

constexpr int kTabWords = 16 + 256; // h[4], l[4], f, pad | table of 256 entries for depth >= 5
constexpr int kMaxPairs = 2048;     // T*k per call
constexpr int kMaxBlocksPerUnit = 4;
constexpr int kMaxMembers = 2;      // tokens per column block: 3 byte columns each in the 8 of an MMA
// Tensor-core path (tc_batch.cu): experts with at least kTcMinTokens pairs at depth <= kTcMaxLevels
// form units of at most kTcMaxCols pairs.
constexpr int kTcMinTokens = 8;
constexpr int kTcMaxLevels = 4;
constexpr int kTcMaxCols = 64;

// Operand rows of the tensor-core units of a call with P pairs: every unit holds >= kTcMinTokens
// pairs and pads them to a multiple of 16 rows.
__host__ __device__ inline int tc_max_rows(int P) { return P + 15 * (P / kTcMinTokens) + 16; }

// Row stride (ints) of the h-fragment exponents: I/128 rounded up to 16 bytes.
__host__ __device__ inline int hexp_stride(int I) { return ((I / 128) + 3) & ~3; }

// flags[] words
constexpr int kFlagError = 0;  // nonzero: error code (see layer.cu)
constexpr int kFlagBlocks = 1; // column blocks
constexpr int kFlagUnits = 2;  // expert units
constexpr int kFlagSched = 3;  // work counter of the persistent kernel
constexpr int kFlagWhere = 4;  // detail of the first error
constexpr int kFlagTcUnits = 8; // tensor-core units of the call
constexpr int kFlagTcRows = 9;  // their operand rows (pairs and padding)

// Device pointers into one layer workspace (see carve_layer_ws).
struct LayerWs {
    int *flags;      // [64]
    int *blk_depth;  // per column block (<= 2 pairs of one expert and one depth): depth
    int *blk_nmem;   //   members (<= kMaxMembers)
    int *blk_pair;   //   [4] pair index t*k + i of each member
    int *blk_expert; //   expert
    int *unit_expert, *unit_blk0, *unit_nblk, *unit_bmax; // per unit (one expert, <= 4 blocks)
    int *utab;       // per unit, 12 ints: expert, bmax, blk0, nblk, slot of planes 0..7
    int *cntA;       // per gate/up item (unit, 16 rows of I): consumer warps finished
    int *cntH;       // per (unit, 128 rows of I): gate/up items finished (8 per tile)
    int *readyB;     // per unit: 128-row tiles of h turned into fragments
    int *cntB;       // per down item (unit, 128 rows of H): consumer warps finished
    int *ycnt;       // [T][H/128]: pairs of a token whose down rows are written
    float *pA;       // [pairs][I/16][8][2][16]: gate/up partial sums per K-part
    float *pB;       // [pairs][H/16][2][16]: down partial sums per K-part
    uint32_t *tabs;  // [pairs][3][kTabWords]: decode tables per block and matrix
    uint32_t *xfrag; // [T][H/32][24]: activation fragments (xfrag.cuh)
    int *xexp;       // [T][H/128]
    float *h;        // [pairs][I]
    uint32_t *hfrag; // [pairs][I/32][24]
    int *hexp;       // [pairs][hexp_stride(I)]
    float *part;     // [pairs][H]: down-projection output of each pair
    // tensor-core path (T >= kTcMinTokens; null otherwise)
    int4 *tc_unit;   // per unit: expert, pairs n, npad | levels << 16, first operand row
    int *tc_rpair;   // per operand row: pair, or -1 for padding
    int *tc_rdep;    //   depth of the pair (0 for padding)
    int *tc_runit;   //   unit
    int *tc_rxe;     //   power-of-two exponent of the row's x operand
    int *tc_rhe;     //   ... of its h operand
    uint16_t *tc_xb; // [rows][H] f16 x operands, per unit in k-step blocks (umma.cuh layout)
    uint16_t *tc_hb; // [rows][I] f16 h operands
    float *tc_gu;    // [pairs][2][I] gate and up rows of tensor-core pairs
    int32_t *ids;    // [pairs]: routing results kept by the decode step
    float *w;
    uint8_t *depth;
};

LayerWs carve_layer_ws(void *ws, int T, int k, int H, int I, size_t *bytes);
pmoe_status check_layer(const pmoe_layer *L, int T, int k);
// Enqueues the prep and persistent kernels of one layer call on stream st.
// logits == nullptr: ids/w/depth are inputs; otherwise they are written.
pmoe_status launch_layer(const pmoe_layer *L, const float *logits, const float *sens, const uint16_t *x,
                         int32_t *ids, float *w, uint8_t *depth, int T, int k, int B, float *y, void *ws,
                         size_t ws_bytes, cudaStream_t st);

// The tensor-core units of a call (after the prep kernel): operands, gate/up, h, down and combine.
pmoe_status launch_tc(const pmoe_layer *L, const uint16_t *x, const float *wts, int T, int k, float *y,
                      const LayerWs &W, cudaStream_t st);
// Limit of every bounded wait inside the layer kernels (one deadline per launch).
void set_wait_limit_ns(uint64_t ns);
uint64_t wait_limit_ns();

} // namespace pmoe
