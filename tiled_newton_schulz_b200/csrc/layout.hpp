// layout.hpp -- host/device shared plain-old-data tables of one planned call.
#pragma once
#include <stdint.h>

namespace himuon {

// Host-side count of kernels enqueued by the library (defined in api.cu).
void count_launch();

// Roles a matrix plays in a call.
enum Role : int { kRoleIn = 0,   // NS input; momentum M (read, then M' written back)
                  kRoleOut = 1,  // NS output; update O of a momentum step
                  kRoleG = 2,    // gradient G of a momentum step
                  kRoleW = 3,    // weights W of a momentum step
                  kNumRoles = 4 };

// One (sub)matrix after the CMuon split; tiles of it are numbered
// tile_begin .. tile_begin + tiles_r * tiles_c - 1, row-major.
struct DevBlock {
  int64_t tile_begin;
  int32_t tiles_r, tiles_c;
  int32_t rows, cols;          // block extent
  int32_t T;                   // tile edge used for this block
  int32_t mat;                 // index of the parent matrix in the call
  int32_t tmap[kNumRoles];     // tensor-map index per role (-1: role absent)
  void *ptr[kNumRoles];        // element (0,0) of the block per role (nullptr: absent)
  int64_t ld[kNumRoles];       // row pitch in elements per role
  int32_t dtype[kNumRoles];    // himuon_dtype per role
};

// One tile of the staged (HBM) path.
struct DevTile {
  int32_t block;               // index into the DevBlock table
  int32_t transposed;          // 1 when the tile is taller than wide
  int32_t r0, c0;              // origin inside the block
  int32_t h, w;                // extent (ragged edge tiles are smaller than T)
};

}  // namespace himuon
