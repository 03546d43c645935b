// fa_seqpar.cu -- fa_weight_partial: the softmax piece of one key window
// rescaled so that the pieces of all windows add up to the output.
//
// "FlashAttention for Efficient Training", section 5.3 (Sequence Parallelism
// for Long Contexts), with the merge identity of section 6.1: for pieces
// (O_s, lse_s) over disjoint key windows, lse = ln sum_s e^lse_s and
// O = sum_s e^(lse_s - lse) O_s.  A rank that holds piece s and every lse_s
// (a small all-gather) can form its term e^(lse_s - lse) O_s alone; the terms
// of all ranks then meet in one sum (an all-reduce) instead of each rank
// gathering and merging every piece.
//
// A warp takes 32 rows: lane l reduces the num_parts logsumexps of row l
// (max, then the sum of exponentials; no shuffles, coalesced across lanes),
// then the warp rescales the 32 rows in place, each lane d/32 floats of a row
// with that row's weight taken from its lane.  Memory-bound: the piece is
// read and written once (at long8k, B=2 H=16 N=8192 d=128: 128 MiB each way).
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/fa.h"

namespace {

constexpr int kWarpsPerBlock = 8;

template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    weight_partial_kernel(float* __restrict__ part_o, const float* __restrict__ all_lse, int num_parts, int part,
                          float* __restrict__ lse_out, long long rows) {
  constexpr int kPer = D / 32;  // floats of a row per lane
  constexpr int kBatch = 8;     // rows loaded before any is stored
  const int lane = threadIdx.x & 31;
  const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long r0 = warp0 * 32; r0 < rows; r0 += nwarps * 32) {
    // lane l reduces the logsumexps of row r0 + l (consecutive lanes read
    // consecutive rows of each piece)
    const long long rl = r0 + lane;
    float w = 0.f;
    if (rl < rows) {
      float mx = -INFINITY;
      for (int s = 0; s < num_parts; ++s) mx = fmaxf(mx, all_lse[(long long)s * rows + rl]);
      float lse = -INFINITY;
      if (mx != -INFINITY) {
        float sum = 0.f;
        for (int s = 0; s < num_parts; ++s) {
          const float ls = all_lse[(long long)s * rows + rl];
          sum += ls == -INFINITY ? 0.f : expf(ls - mx);
        }
        lse = mx + logf(sum);
        const float mine = all_lse[(long long)part * rows + rl];
        w = mine == -INFINITY ? 0.f : expf(mine - lse);
      }
      if (lse_out) lse_out[rl] = lse;
    }
    // then the warp rescales its rows, each lane d/32 floats of every row,
    // kBatch rows in flight at a time
    const int nr = rows - r0 < 32 ? (int)(rows - r0) : 32;
    for (int j0 = 0; j0 < nr; j0 += kBatch) {
      float v[kBatch][kPer];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (j0 + j < nr) {
          const float* row = part_o + (r0 + j0 + j) * D + lane * kPer;
          if constexpr (kPer == 4) {
            const float4 t = *reinterpret_cast<const float4*>(row);
            v[j][0] = t.x, v[j][1] = t.y, v[j][2] = t.z, v[j][3] = t.w;
          } else {
            const float2 t = *reinterpret_cast<const float2*>(row);
            v[j][0] = t.x, v[j][1] = t.y;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, (j0 + j) & 31);
        if (j0 + j < nr) {
          float* row = part_o + (r0 + j0 + j) * D + lane * kPer;
          if constexpr (kPer == 4)
            *reinterpret_cast<float4*>(row) = make_float4(v[j][0] * wj, v[j][1] * wj, v[j][2] * wj, v[j][3] * wj);
          else
            *reinterpret_cast<float2*>(row) = make_float2(v[j][0] * wj, v[j][1] * wj);
        }
      }
    }
  }
}

}  // namespace

extern "C" int fa_weight_partial(float* part_o, const float* all_lse, int num_parts, int part, float* lse, int B,
                                 int H, int N, int d, void* stream) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (num_parts < 1 || num_parts > 4096 || part < 0 || part >= num_parts) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return FA_OK;
  if (!part_o || !all_lse) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(part_o) & 15u) || (reinterpret_cast<uintptr_t>(all_lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGNMENT;
  const long long rows = (long long)B * H * N;
  if (rows * num_parts > (1ll << 40)) return FA_ERR_TOO_LARGE;
  const long long want = (rows + 32 * kWarpsPerBlock - 1) / (32 * kWarpsPerBlock);
  const int grid = (int)(want < 148 * 16 ? want : 148 * 16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64)
    weight_partial_kernel<64><<<grid, kWarpsPerBlock * 32, 0, st>>>(part_o, all_lse, num_parts, part, lse, rows);
  else
    weight_partial_kernel<128><<<grid, kWarpsPerBlock * 32, 0, st>>>(part_o, all_lse, num_parts, part, lse, rows);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
