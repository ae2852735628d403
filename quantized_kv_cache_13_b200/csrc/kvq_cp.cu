// kvq_cp.cu -- merging decode attention computed over disjoint parts of each
// sequence (context parallelism: every GPU holds its own part of the cache).
//
// Part r of a row (one query head of one sequence) gives its normalised
// output o_r[D] and the log-sum-exp lse_r of its scores.  Over the union of
// the parts, exp(lse) = sum_r exp(lse_r) and o = sum_r exp(lse_r - lse) o_r:
// the log-sum-exp merge of split-K flash decoding, applied across devices
// after the parts' records have been gathered (an all-gather over NCCL).  A
// part without keys has lse_r = -inf and no weight.
#include <cuda_runtime.h>
#include <math.h>

#include "kvq.h"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int D = kHeadDim;

// One thread per (row, head_dim element); each thread rereads the row's n
// log-sum-exps (n is small: the number of devices).
__global__ void __launch_bounds__(256) combine_kernel(int n, int64_t rows, const float* o_parts,
                                                     int64_t o_stride, const float* lse_parts,
                                                     int64_t lse_stride, float* out,
                                                     float* lse_out) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * D) return;
  const int64_t row = idx / D;
  const int d = (int)(idx % D);
  float m = -INFINITY;
  for (int r = 0; r < n; ++r) m = fmaxf(m, lse_parts[r * lse_stride + row]);
  if (m == -INFINITY) {   // no part holds a key
    out[idx] = 0.0f;
    if (lse_out && d == 0) lse_out[row] = -INFINITY;
    return;
  }
  float acc = 0.0f, wsum = 0.0f;
  for (int r = 0; r < n; ++r) {
    const float lr = lse_parts[r * lse_stride + row];
    const float w = (lr == -INFINITY) ? 0.0f : expf(lr - m);
    wsum += w;
    acc += w * o_parts[r * o_stride + row * D + d];
  }
  out[idx] = acc / wsum;
  if (lse_out && d == 0) lse_out[row] = m + logf(wsum);
}

// The result of attention over no keys: o = 0, lse = -inf.
__global__ void __launch_bounds__(256) empty_part_kernel(int64_t rows, float* out, float* lse) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * D) return;
  out[idx] = 0.0f;
  if (lse && idx % D == 0) lse[idx / D] = -INFINITY;
}

unsigned blocks_for(int64_t threads) { return (unsigned)((threads + 255) / 256); }

}  // namespace

cudaError_t launch_combine(int n, int64_t rows, const float* o_parts, int64_t o_stride,
                           const float* lse_parts, int64_t lse_stride, float* out, float* lse_out,
                           cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  combine_kernel<<<blocks_for(rows * D), 256, 0, stream>>>(n, rows, o_parts, o_stride, lse_parts,
                                                           lse_stride, out, lse_out);
  return cudaGetLastError();
}

cudaError_t launch_empty_part(int64_t rows, float* out, float* lse, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  empty_part_kernel<<<blocks_for(rows * D), 256, 0, stream>>>(rows, out, lse);
  return cudaGetLastError();
}

}  // namespace kvq
