// Device twin of workload/gen.py: SplitMix64 outputs mapped through the host-built 65536-entry
// bf16 N(0,1) quantile table.  Output i of a stream with key k is mix64(k + (i + 1) * GAMMA)
// (Steele, Lea & Flood, OOPSLA 2014); the value is table[output >> 48].  Integer arithmetic and
// a table lookup only, so every value equals the host generator's bit for bit.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint32_t draw(uint64_t key, uint64_t i, const uint16_t* table) {
  return table[mix64(key + (i + 1) * kGamma) >> 48];
}

__global__ void fill_normal_kernel(uint16_t* out, int64_t n, uint64_t key, uint64_t start,
                                   const uint16_t* table) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (uint16_t)draw(key, start + (uint64_t)i, table);
}

// Prefill of one layer's paged pool: token j of sequence b (j < n_tokens[b]) gets the values
// (j*Hkv + h)*128 + d of stream keys[b], stored at page page_table[b][j/16], slot j%16.
// One thread writes 8 consecutive dims (16 bytes).  Entries outside the pool are skipped.
__global__ void fill_kv_kernel(uint16_t* pool, const int32_t* page_table, int max_pages, int Hkv,
                               const int32_t* n_tokens, const uint64_t* keys, int64_t n_pool_pages,
                               const uint16_t* table) {
  const int b = blockIdx.y;
  const int64_t n = n_tokens[b];
  const uint64_t key = keys[b];
  const int64_t per_tok = (int64_t)Hkv * 16;   // 8-dim groups per token
  const int64_t total = n * per_tok;
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = w / per_tok;
    const int rem = (int)(w - j * per_tok);
    const int h = rem >> 4, g8 = rem & 15;
    const int64_t phys = page_table[(int64_t)b * max_pages + j / 16];
    if (phys < 0 || phys >= n_pool_pages) continue;
    const uint64_t base = (uint64_t)((j * Hkv + h) * 128 + g8 * 8);
    uint4 v;
    v.x = draw(key, base + 0, table) | (draw(key, base + 1, table) << 16);
    v.y = draw(key, base + 2, table) | (draw(key, base + 3, table) << 16);
    v.z = draw(key, base + 4, table) | (draw(key, base + 5, table) << 16);
    v.w = draw(key, base + 6, table) | (draw(key, base + 7, table) << 16);
    uint4* dst = reinterpret_cast<uint4*>(pool + (((phys * Hkv + h) * 16 + (j % 16)) * 128 + g8 * 8));
    *dst = v;
  }
}

}  // namespace

extern "C" {

// out[i] = bf16 N(0,1) draw start+i of stream `key`, i < n.  Returns a cudaError_t.
int odagen_fill_normal_bf16(uint16_t* out, int64_t n, uint64_t key, uint64_t start,
                            const uint16_t* table, cudaStream_t stream) {
  if (n <= 0) return 0;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 65535 * 4) blocks = 65535 * 4;
  fill_normal_kernel<<<(unsigned)blocks, 256, 0, stream>>>(out, n, key, start, table);
  return (int)cudaGetLastError();
}

// Prefill of a paged pool [n_pool_pages][Hkv][16][128] bf16 for B sequences (device arrays
// n_tokens[B], keys[B], page_table[B][max_pages]).  Returns a cudaError_t.
int odagen_fill_kv(uint16_t* pool, const int32_t* page_table, int B, int max_pages, int Hkv,
                   const int32_t* n_tokens, const uint64_t* keys, int64_t max_tokens,
                   int64_t n_pool_pages, const uint16_t* table, cudaStream_t stream) {
  if (B <= 0 || max_tokens <= 0) return 0;
  int64_t groups = max_tokens * Hkv * 16;
  int64_t bx = (groups + 255) / 256;
  if (bx > 8192) bx = 8192;
  fill_kv_kernel<<<dim3((unsigned)bx, (unsigned)B), 256, 0, stream>>>(
      pool, page_table, max_pages, Hkv, n_tokens, keys, n_pool_pages, table);
  return (int)cudaGetLastError();
}

}  // extern "C"
