// Read-bandwidth probe: the L2 denominator of the draft's roofline.
//
// The draft streams the rank-r factor Bf [r,V] once per position; when few
// requests share a position (one request at K = 16) almost all of those reads
// are served by L2 rather than HBM, so the draft's Bf read rate is compared
// with the rate plain loads draw from an L2-resident buffer. This is not part
// of the library's path: it lives in its own shared object, which only the
// benchmark loads.
//
// One persistent grid (four 512-thread CTAs per SM) reads a device buffer
// `passes` times with 16-byte loads cached at L2 only (ld.global.cg), four
// independent loads in flight per thread, and folds the data into one word per
// thread written to `sink`, so that no load can be removed. A buffer well
// below the L2's capacity (126 MB on B200) stays resident after the first pass.
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace {

constexpr int kBlock = 512;
constexpr int kCtasPerSm = 4;

__device__ __forceinline__ unsigned fold(const uint4& v) { return v.x ^ v.y ^ v.z ^ v.w; }

__global__ void __launch_bounds__(kBlock, kCtasPerSm) l2_read_kernel(const uint4* __restrict__ buf, int n16, int passes,
                                                                     unsigned* __restrict__ sink) {
  const int stride = gridDim.x * blockDim.x;
  const int i0 = blockIdx.x * blockDim.x + threadIdx.x;
  unsigned a0 = 0, a1 = 0, a2 = 0, a3 = 0;
  for (int p = 0; p < passes; ++p) {
    int i = i0;
    for (; i < n16 - 3 * stride; i += 4 * stride) {
      const uint4* q = buf + i;
      const uint4 x0 = __ldcg(q);
      const uint4 x1 = __ldcg(q + stride);
      const uint4 x2 = __ldcg(q + 2 * stride);
      const uint4 x3 = __ldcg(q + 3 * stride);
      a0 ^= fold(x0);
      a1 ^= fold(x1);
      a2 ^= fold(x2);
      a3 ^= fold(x3);
    }
    for (; i < n16; i += stride) a0 ^= fold(__ldcg(buf + i));
  }
  sink[i0] = a0 ^ a1 ^ a2 ^ a3;
}

}  // namespace

extern "C" {

// Words of `sink` that dspark_probe_l2_read writes on the current device (one
// per thread of its grid), or 0 if the device cannot be queried.
size_t dspark_probe_sink_words(void) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return static_cast<size_t>(sms) * kCtasPerSm * kBlock;
}

// Reads `bytes` of device memory at `buf` `passes` times on `stream`
// (asynchronous). buf: 16-byte aligned; bytes: a positive multiple of 16;
// passes >= 1; sink: device memory of at least dspark_probe_sink_words()
// 32-bit words, overwritten. Returns 0 on success, 1 for an invalid argument
// (nothing launched), 3 for a CUDA error.
int dspark_probe_l2_read(const void* buf, size_t bytes, int passes, unsigned* sink, size_t sink_words,
                         void* stream) {
  const size_t words = dspark_probe_sink_words();
  if (buf == nullptr || sink == nullptr || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0) return 1;
  if (bytes == 0 || bytes % 16 != 0 || passes < 1 || words == 0 || sink_words < words) return 1;
  if (bytes / 16 > static_cast<size_t>(1) << 30) return 1;  // 32-bit indices, with room for 4 strides
  const int grid = static_cast<int>(words / kBlock);
  l2_read_kernel<<<grid, kBlock, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(buf), static_cast<int>(bytes / 16), passes, sink);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

}  // extern "C"
