// Backward pass: the state transpose the three sweeps need.
//
// The gradients of o_t = q_t S_t, S_t = lambda S_{t-1} + k_t^T v_t (for a loss
// with gradients dO of the outputs and dS_N of the final state) are three runs
// of the same chunked recurrence with the roles of q, k, v exchanged:
//   dq: forward in time, q <- dO, k <- v, v <- k, initial state S0^T;
//   dk: backward in time, q <- v, k <- dO, v <- q, initial state dS_N^T;
//   dv: backward in time, q <- k, k <- q, v <- dO, initial state dS_N, whose
//       final state is dS_0.
// Only the transposed states are new; this kernel writes them.
#pragma once

#include "la_ptx.cuh"

namespace la {

constexpr int kTransposeTile = 32;

// dst[m][j][i] = src[m][i][j] for m in [0, count) D x D fp32 matrices. Grid (D/32, D/32, count),
// block (32, 8): a 32 x 32 tile through shared memory (padded rows, no bank conflicts).
__global__ void __launch_bounds__(256) la_transpose_states_kernel(const float *src, float *dst, int D) {
    __shared__ float tile[kTransposeTile][kTransposeTile + 1];
    const size_t base = static_cast<size_t>(blockIdx.z) * D * D;
    const int bx = blockIdx.x * kTransposeTile, by = blockIdx.y * kTransposeTile;
    for (int r = threadIdx.y; r < kTransposeTile; r += blockDim.y)
        tile[r][threadIdx.x] = src[base + static_cast<size_t>(by + r) * D + bx + threadIdx.x];
    __syncthreads();
    for (int r = threadIdx.y; r < kTransposeTile; r += blockDim.y)
        dst[base + static_cast<size_t>(bx + r) * D + by + threadIdx.x] = tile[threadIdx.x][r];
}

}  // namespace la
