// Page movement: whole page records (all kv heads of one physical page,
// num_kv_heads * block bytes contiguous bytes) gathered out of the pool, scattered
// back into it, copied inside it, and residual rows copied between batch
// rows.  These are the operations a paged cache needs to swap sequences out
// to host memory and back and to fork a sequence copy-on-write ("KV-Cache
// und PagedAttention: Warum Ihr LLM-Server langsamer wird", "Wie
// PagedAttention das loest": pages are allocated on demand, shared between
// sequences and copied only when written).
//
// The copy is bound by HBM bandwidth: each CTA takes whole records in turn
// and moves them with 16-byte loads and stores, four in flight per thread.
#include "kernels.cuh"

namespace s4kv {

namespace {
constexpr int kMoveThreads = 256;
constexpr int kMoveUnroll = 4;
}  // namespace

__global__ void __launch_bounds__(kMoveThreads) move_kernel(const MoveParams p) {
  const long long vecs = p.rec_bytes / 16;
  for (int i = blockIdx.x; i < p.n; i += gridDim.x) {
    const int si = p.src_idx ? __ldg(p.src_idx + i) : i;
    const int di = p.dst_idx ? __ldg(p.dst_idx + i) : i;
    if (static_cast<unsigned>(si) >= static_cast<unsigned>(p.src_limit) ||
        static_cast<unsigned>(di) >= static_cast<unsigned>(p.dst_limit)) {
      if (threadIdx.x == 0) flag_error(p.err, p.err_bit);
      continue;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(p.src_base + si * p.rec_bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(p.dst_base + di * p.rec_bytes);
    long long k = threadIdx.x;
    for (; k + (kMoveUnroll - 1) * kMoveThreads < vecs; k += kMoveUnroll * kMoveThreads) {
      uint4 v[kMoveUnroll];
#pragma unroll
      for (int u = 0; u < kMoveUnroll; ++u) v[u] = src[k + u * kMoveThreads];
#pragma unroll
      for (int u = 0; u < kMoveUnroll; ++u) dst[k + u * kMoveThreads] = v[u];
    }
    for (; k < vecs; k += kMoveThreads) dst[k] = src[k];
  }
}

void launch_move(const MoveParams &p, cudaStream_t stream) {
  if (p.n <= 0) return;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  const int grid = p.n < 8 * sms ? p.n : 8 * sms;  // 8 resident CTAs of 256 threads per SM
  move_kernel<<<grid, kMoveThreads, 0, stream>>>(p);
}

}  // namespace s4kv
