// Reversal of the sequence axis: dst[bh][S-1-t][:] = src[bh][t][:] for tensors laid out
// [BH, S, D] (D elements of `esize` bytes per token).  Used by the reversed-sequence pass
// (the backward direction of a bidirectional encoder), which runs the forward kernels on
// reversed copies of its inputs and reverses h back.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace mlstm {
namespace {

// one thread per 16-byte word (row bytes a multiple of 16) or per element
template <typename W>
__global__ void reverse_rows_kernel(const W* __restrict__ src, W* __restrict__ dst, long long BH, long long S,
                                    long long words) {
  const long long total = BH * S * words;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long w = i % words, row = i / words;
    const long long t = row % S, bh = row / S;
    dst[(bh * S + (S - 1 - t)) * words + w] = src[i];
  }
}

}  // namespace

cudaError_t launch_reverse_rows(const void* src, void* dst, long long BH, long long S, long long row_bytes,
                                cudaStream_t stream) {
  if (BH == 0 || S == 0 || row_bytes == 0) return cudaSuccess;
  const int threads = 256;
  if (row_bytes % 16 == 0 && ((uintptr_t)src & 15) == 0 && ((uintptr_t)dst & 15) == 0) {
    const long long words = row_bytes / 16, total = BH * S * words;
    const int blocks = (int)((total + threads - 1) / threads < 148 * 16 ? (total + threads - 1) / threads : 148 * 16);
    reverse_rows_kernel<uint4><<<blocks, threads, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                                BH, S, words);
  } else if (row_bytes % 4 == 0) {
    const long long words = row_bytes / 4, total = BH * S * words;
    const int blocks = (int)((total + threads - 1) / threads < 148 * 16 ? (total + threads - 1) / threads : 148 * 16);
    reverse_rows_kernel<uint32_t><<<blocks, threads, 0, stream>>>(static_cast<const uint32_t*>(src),
                                                                   static_cast<uint32_t*>(dst), BH, S, words);
  } else {
    const long long words = row_bytes / 2, total = BH * S * words;
    const int blocks = (int)((total + threads - 1) / threads < 148 * 16 ? (total + threads - 1) / threads : 148 * 16);
    reverse_rows_kernel<uint16_t><<<blocks, threads, 0, stream>>>(static_cast<const uint16_t*>(src),
                                                                   static_cast<uint16_t*>(dst), BH, S, words);
  }
  return cudaGetLastError();
}

}  // namespace mlstm
