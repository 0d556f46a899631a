// Streaming-read ceiling kernels: how fast can a B200 read a large buffer
// once, with the access shapes the GEMV kernels can use. They move the same
// bytes a decode GEMV streams and only fold them into a checksum, so their
// rate is the read ceiling the GEMV is measured against.
//
//   mode 0: 16-byte global loads per thread, `depth` loads in flight per thread;
//   mode 1: 1-D bulk async copies (TMA bulk engine) of `chunk` bytes into a
//           per-warp ring of `depth` shared-memory stages, each warp reading
//           its contiguous share of the buffer;
//   mode 2: as mode 1 with one ring per CTA (one elected thread issues copies
//           for the whole CTA, the warps read disjoint parts of each stage).
#include <cuda_runtime.h>

#include "tern_ptx.cuh"

namespace tern {

int read_clear_dev_error_stream(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

template <int DEPTH>
__global__ void __launch_bounds__(512) stream_ldg_kernel(const uint4* __restrict__ src, size_t n16,
                                                         unsigned* __restrict__ sink) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + (DEPTH - 1) * stride < n16; i += DEPTH * stride) {
    uint4 v[DEPTH];
#pragma unroll
    for (int d = 0; d < DEPTH; ++d) v[d] = __ldcs(src + i + d * stride);
#pragma unroll
    for (int d = 0; d < DEPTH; ++d) acc ^= v[d].x ^ v[d].y ^ v[d].z ^ v[d].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldcs(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  if (acc == 0x9E3779B9u) atomicAdd(sink, 1u);  // keeps the loads alive
}

// Each warp (mode 1) or CTA (mode 2) owns a contiguous range of the buffer
// and streams it through `depth` stages of `chunk` bytes.
__global__ void __launch_bounds__(512) stream_bulk_kernel(const uint8_t* __restrict__ src, size_t bytes, int chunk,
                                                          int depth, int per_warp, unsigned* __restrict__ sink) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int owners_per_cta = per_warp ? nw : 1;
  const int owner = per_warp ? warp : 0;
  const size_t n_owner = (size_t)gridDim.x * owners_per_cta;
  const size_t gid = (size_t)blockIdx.x * owners_per_cta + owner;
  const size_t nchunks = bytes / chunk;
  const size_t c0 = nchunks * gid / n_owner, c1 = nchunks * (gid + 1) / n_owner;
  const int nst = (int)(c1 - c0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem) + owner * depth;
  uint8_t* ring = smem + ((size_t)owners_per_cta * depth * 8 + 127) / 128 * 128 + (size_t)owner * depth * chunk;
  const bool issuer = per_warp ? lane == 0 : threadIdx.x == 0;
  if (issuer) {
    for (int s = 0; s < depth; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  if (per_warp) __syncwarp(); else __syncthreads();
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int i) {
    const int slot = i % depth;
    mbar_arrive_expect_tx(&bars[slot], (uint32_t)chunk);
    bulk_g2s(ring + (size_t)slot * chunk, src + (c0 + i) * (size_t)chunk, (uint32_t)chunk, &bars[slot], pol);
  };
  if (issuer)
    for (int i = 0; i < min(depth, nst); ++i) issue(i);
  uint32_t acc = 0;
  const int readers = per_warp ? 32 : blockDim.x;
  const int rid = per_warp ? lane : threadIdx.x;
  bool ok = true;
  for (int i = 0; i < nst && ok; ++i) {
    const int slot = i % depth;
    ok = mbar_wait_bounded(&bars[slot], (uint32_t)(i / depth) & 1u);
    if (per_warp) ok = __all_sync(0xffffffffu, ok); else ok = __syncthreads_and(ok);
    if (!ok) break;
    const uint4* st = reinterpret_cast<const uint4*>(ring + (size_t)slot * chunk);
    for (int j = rid; j < chunk / 16; j += readers) {
      const uint4 v = st[j];
      acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    fence_proxy_async_smem();
    if (per_warp) __syncwarp(); else __syncthreads();
    if (issuer && i + depth < nst) issue(i + depth);
  }
  if (acc == 0x9E3779B9u) atomicAdd(sink, 1u);
}

}  // namespace

// Returns 0 on success, -1 for an invalid request, else a CUDA error code.
int launch_stream_read(const void* src, size_t bytes, int mode, int chunk, int depth, int ctas_per_sm, int warps,
                       unsigned* sink, void* stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (warps < 1 || warps > 16 || ctas_per_sm < 1 || ctas_per_sm > 32) return -1;
  if (mode == 0) {
    if ((reinterpret_cast<uintptr_t>(src) & 15u) || bytes % 16) return -1;
    const dim3 grid(sms * ctas_per_sm), block(32 * warps);
    const size_t n16 = bytes / 16;
    const uint4* p = static_cast<const uint4*>(src);
    switch (depth) {
      case 1: stream_ldg_kernel<1><<<grid, block, 0, s>>>(p, n16, sink); break;
      case 2: stream_ldg_kernel<2><<<grid, block, 0, s>>>(p, n16, sink); break;
      case 4: stream_ldg_kernel<4><<<grid, block, 0, s>>>(p, n16, sink); break;
      case 8: stream_ldg_kernel<8><<<grid, block, 0, s>>>(p, n16, sink); break;
      default: return -1;
    }
    return (int)cudaGetLastError();
  }
  if (mode != 1 && mode != 2) return -1;
  if (chunk < 16 || chunk % 16 || depth < 1 || depth > 16 || (reinterpret_cast<uintptr_t>(src) & 15u)) return -1;
  const int owners = mode == 1 ? warps : 1;
  const size_t smem = ((size_t)owners * depth * 8 + 127) / 128 * 128 + (size_t)owners * depth * chunk;
  if (smem > 227 * 1024) return -1;
  cudaError_t e = cudaFuncSetAttribute(stream_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  stream_bulk_kernel<<<sms * ctas_per_sm, 32 * warps, smem, s>>>(static_cast<const uint8_t*>(src), bytes, chunk, depth,
                                                                 mode == 1, sink);
  return (int)cudaGetLastError();
}

}  // namespace tern
