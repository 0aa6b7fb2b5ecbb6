// Workspace layout of the layer kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/pmoe.h"

namespace pmoe {

constexpr int kTabWords = 16 + 256; // h[4], l[4], f, pad | shared-memory table of 256 entries
constexpr int kFlagError = 0, kFlagBlocks = 1, kFlagUnits = 2;
constexpr int kMaxPairs = 2048;

// Device pointers into one layer workspace (see carve_layer_ws).
struct LayerWs {
    int *flags;      // [64]: error, number of blocks, number of units
    int *blk_depth;  // per column block: depth
    int *blk_nmem;   //   members (1..4)
    int *blk_pair;   //   [4] pair index t*k + i of each member
    int *blk_expert; //   expert
    int *unit_expert, *unit_blk0, *unit_nblk, *unit_bmax; // per unit (expert, <= 8 blocks)
    uint32_t *tabs;  // [pairs][3][kTabWords]: decode tables per block and matrix
    uint32_t *xfrag; // [T][H/32][8][2]
    int *xexp;       // [T][H/128]
    float *h;        // [pairs][I]
    uint32_t *hfrag; // [pairs][I/32][8][2]
    int *hexp;       // [pairs][I/128]
    float *part;     // [pairs][H]: down-projection output of each pair
    int32_t *ids;    // [pairs]: routing results kept by the decode step
    float *w;
    uint8_t *depth;
};

LayerWs carve_layer_ws(void *ws, int T, int k, int H, int I, size_t *bytes);
pmoe_status check_layer(const pmoe_layer *L, int T, int k);

} // namespace pmoe
