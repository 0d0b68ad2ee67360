// resident.hpp -- launch interface of the on-chip (T <= 128) tiled NS kernel.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.hpp"

namespace himuon {

constexpr int kMaxSteps = 16;

// Per-step scalars derived on the host from (a_t, b_t, c_t); see
// make_resident_steps() for their meaning.  The iterate is carried scaled,
// as gamma_t X_t, so that S needs no scaling of its own (s = 1).
struct ResidentStep {
  float s;          // S = r(s * D_P) feeds MMA2
  float beta;       // Bop = r(beta * D_P + a * I) feeds MMA3
  float a;          // a_t
  float xr;         // next operand r(xr * D_X) = gamma_{t+1} X_{t+1}  (xr = gamma_{t+1} / gamma_t)
  uint32_t neg2;    // MMA2 negates its A operand (c_t / beta < 0)
  uint32_t acc2;    // MMA2 accumulates onto A (b_t != 0)
};

struct ResidentArgs {
  const DevBlock *blocks;
  const CUtensorMap *tmaps;
  int32_t n_blocks;
  int32_t K;
  int64_t n_tiles;
  int32_t mode;     // 0: NS in -> out; 1: momentum step
  int32_t has_w, has_o;
  int32_t op_fmt;   // tensor-core operand type: 0 fp16, 1 bf16
  int32_t f16_small;  // bf16 call: super-tiles of tiles with short side <= 64 use fp16 operands
  int32_t smem_blocks;  // 1: the block table fits the kernel's compact shared-memory copy
  int32_t pack;     // tiles per 128 x 128 super-tile: 1 (T = 128), 2 (T = 64) or 4 (T = 32)
  int32_t test_stall;  // self-test: CTA 0 waits on a barrier nothing arrives on (timeout path)
  float mu, lr, eps, safety;
  float gamma0;     // X_0 operand = r(gamma0 M' / rho)
  float oscale;     // O = oscale * D_X after the last step (1 / gamma_{K-1})
  ResidentStep step[kMaxSteps];
  int *status;
};

// Fills args.step[0..K) from K coefficient triples.
void make_resident_steps(ResidentArgs &args, const float *coeffs, int K);

int resident_smem_bytes();
// 256 x 256 tiles on CTA pairs (clusters of two): `pairs` tiles in flight.
int pair_smem_bytes();
cudaError_t launch_ns_pair(const ResidentArgs &args, int pairs, cudaStream_t stream);
int resident_max_smem_blocks();
cudaError_t launch_ns_resident(const ResidentArgs &args, int grid, cudaStream_t stream);

}  // namespace himuon
