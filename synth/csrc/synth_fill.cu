// Device-side fills for the seeded synthetic inputs.
//
// Implements exactly the definition in synth/gen.py: value = table[top 16
// bits of mix64(key + counter)], mix64 being the SplitMix64 output function
// (Steele, Lea & Flood, OOPSLA 2014). Integer arithmetic and a table lookup
// only, so the bytes match the numpy generator bit for bit. Holds no
// arithmetic of the attention method; the paged fill only knows where a
// (layer, row, head, K/V, position) lands in the paged cache layout.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

template <typename E>
__global__ void fill_streams_kernel(E* dst, const uint64_t* keys, const uint64_t* offs, int ns,
                                    long long n_outer, long long inner, const E* table) {
  const long long total = (long long)ns * n_outer * inner;
  for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < total;
       it += (long long)gridDim.x * blockDim.x) {
    const long long j = it % inner;
    const long long r = it / inner;
    const int s = (int)(r % ns);
    const long long i = r / ns;
    const uint64_t c = keys[s] + offs[s] + (uint64_t)(i * inner + j);
    dst[it] = table[mix64(c) >> 48];
  }
}

template <typename E>
__global__ void fill_paged_kernel(E* cache, const uint64_t* keys, const int32_t* block_table,
                                  const int32_t* npos, int L, int B, int hkv, int d, int bs,
                                  int max_blocks, long long num_blocks, int pmax, const E* table,
                                  int* bad) {
  // one thread per element of every (l, b, g, kv, position) row
  const long long rows = (long long)L * B * hkv * 2 * pmax;
  const long long total = rows * d;
  const long long layer_elems = num_blocks * hkv * 2 * (long long)bs * d;
  for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < total;
       it += (long long)gridDim.x * blockDim.x) {
    const int dd = (int)(it % d);
    long long r = it / d;
    const int p0 = (int)(r % pmax); r /= pmax;        // position - 1
    const int kv = (int)(r % 2); r /= 2;
    const int g = (int)(r % hkv); r /= hkv;
    const int b = (int)(r % B); r /= B;
    const int l = (int)r;
    if (p0 >= npos[b]) continue;
    const int bi = p0 / bs;
    const int blk = bi < max_blocks ? block_table[(long long)b * max_blocks + bi] : -1;
    if (blk < 0 || blk >= num_blocks) { atomicExch(bad, 1); continue; }
    const uint64_t key = keys[(((long long)l * B + b) * hkv + g) * 2 + kv];
    const uint64_t c = key + (uint64_t)((long long)p0 * d + dd);
    const long long off = (long long)l * layer_elems +
                          ((((long long)blk * hkv + g) * 2 + kv) * bs + (p0 % bs)) * d + dd;
    cache[off] = table[mix64(c) >> 48];
  }
}

int grid_for(long long n) {
  long long g = (n + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" {

// dst[(i*ns + s)*inner + j] = table[top16(mix64(keys[s] + offs[s] + i*inner + j))]
int synth_fill_streams(void* dst, int elem_bytes, const uint64_t* keys, const uint64_t* offs,
                       int ns, long long n_outer, long long inner, const void* table,
                       void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long n = (long long)ns * n_outer * inner;
  if (n <= 0) return 0;
  if (elem_bytes == 2)
    fill_streams_kernel<uint16_t><<<grid_for(n), 256, 0, st>>>(
        static_cast<uint16_t*>(dst), keys, offs, ns, n_outer, inner,
        static_cast<const uint16_t*>(table));
  else if (elem_bytes == 4)
    fill_streams_kernel<uint32_t><<<grid_for(n), 256, 0, st>>>(
        static_cast<uint32_t*>(dst), keys, offs, ns, n_outer, inner,
        static_cast<const uint32_t*>(table));
  else
    return 1;
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

// Paged cache [L][num_blocks][hkv][2][bs][d]: positions 1..npos[b] of every
// (layer, row, head, K/V) stream; stream key keys[((l*B+b)*hkv+g)*2+kv],
// counter (p-1)*d + dim. `bad` (device int) is set if a table entry is out of range.
int synth_fill_paged_kv(void* cache, int elem_bytes, const uint64_t* keys,
                        const int32_t* block_table, const int32_t* npos, int L, int B, int hkv,
                        int d, int bs, int max_blocks, long long num_blocks, int pmax,
                        const void* table, int* bad, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long n = (long long)L * B * hkv * 2 * pmax * d;
  if (n <= 0) return 0;
  if (elem_bytes == 2)
    fill_paged_kernel<uint16_t><<<grid_for(n), 256, 0, st>>>(
        static_cast<uint16_t*>(cache), keys, block_table, npos, L, B, hkv, d, bs, max_blocks,
        num_blocks, pmax, static_cast<const uint16_t*>(table), bad);
  else if (elem_bytes == 4)
    fill_paged_kernel<uint32_t><<<grid_for(n), 256, 0, st>>>(
        static_cast<uint32_t*>(cache), keys, block_table, npos, L, B, hkv, d, bs, max_blocks,
        num_blocks, pmax, static_cast<const uint32_t*>(table), bad);
  else
    return 1;
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // extern "C"
