// selector_microbench.cu -- the selector's per-block work in isolation.
//
// Times, on shared-memory-resident 64-token int4 scan tiles, the work one warp
// does per key block in the decode kernel's selector: the query fold
// (fold_block), the integer scan (block_best: mma.sync m16n8k32, u8 nibbles x
// s8 query), the block scores (block_scores) and the Top-delta keep test.
// Variants drop one part (no fold, no mma, fold only) or replace the mma scan
// by a dp4a form (lane = token group x channel quarter, two dp4a per packed
// word and head, shuffle sum over the quarters, token max), and the grid is
// varied (1 CTA of 1..8 warps; 296 CTAs = two per SM).  Prints cycles per
// block per warp (clock64) and blocks per us per SM (CUDA events), and the
// cost of __nanosleep.  It includes the kernel source, so the functions timed
// are the shipped ones.
//
// Build and run on a B200 (from the repository root):
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 --expt-relaxed-constexpr \
//        -I include -I sparse_long_context_ffd_b200/csrc \
//        -o /tmp/selector_microbench sparse_long_context_ffd_b200/microbench/selector_microbench.cu
//   /tmp/selector_microbench
#include "../csrc/decode.cu"
#include <cstdio>
#include <vector>

using namespace ffd;

constexpr int T = 64, F = 0, NT = 8;  // 8 resident tiles
constexpr int TILE = T * 64 + 256;

// dp4a form of the per-block integer scan: lane (tg = lane >> 2, c4 = lane & 3)
// takes tokens tg + 8k (k < 8) and channel quarter c4 (packed words 4 c4 .. 4 c4 + 3);
// qe/qo hold the int8 query of the even / odd channels of those words per head.
template <int G>
__device__ __forceinline__ void block_best_dp4a(const uint8_t *tile, const uint32_t (&qe)[G][4],
                                                const uint32_t (&qo)[G][4], int lane, int &best0, int &best1) {
  const int tg = lane >> 2, c4 = lane & 3;
  int bh[G];
#pragma unroll
  for (int h = 0; h < G; ++h) bh[h] = INT_MIN;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 w = *reinterpret_cast<const uint4 *>(tile + (tg + 8 * k) * 64 + 16 * c4);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    int acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = ww[i] & 0x0F0F0F0Fu, hi = (ww[i] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        acc[h] = __dp4a(static_cast<int>(lo), static_cast<int>(qe[h][i]), acc[h]);
        acc[h] = __dp4a(static_cast<int>(hi), static_cast<int>(qo[h][i]), acc[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      acc[h] += __shfl_xor_sync(kFull, acc[h], 1);
      acc[h] += __shfl_xor_sync(kFull, acc[h], 2);
      bh[h] = max(bh[h], acc[h]);
    }
  }
  // heads 2 t4, 2 t4 + 1 for the caller's layout (lane & 3)
  best0 = INT_MIN;
  best1 = INT_MIN;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (h == 2 * (lane & 3)) best0 = bh[h];
    if (h == 2 * (lane & 3) + 1) best1 = bh[h];
  }
}

template <int G, int V>
__global__ void scan_bench(const uint8_t *tiles_g, const uint16_t *q, int iters, float *out,
                           long long *cyc) {
  extern __shared__ __align__(16) uint8_t sm[];
  for (int i = threadIdx.x * 16; i < NT * TILE; i += blockDim.x * 16)
    *reinterpret_cast<uint4 *>(sm + i) = *reinterpret_cast<const uint4 *>(tiles_g + i);
  __syncthreads();
  using SF = ScanFold<G, F>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, t4 = lane & 3;
  uint32_t qv[SF::NC / 2];
  SF::load_pairs(q + (gid % G) * 128 + 32 * t4, SF::part(gid), qv);
  volatile uint32_t *qbits = reinterpret_cast<volatile uint32_t *>(sm + NT * TILE) + warp * 64;
  uint32_t bq[8];
  int sq;
  float am;
  fold_block<G, F>(reinterpret_cast<const uint16_t *>(sm + T * 64), qv, lane, bq, sq, am);
  float run0 = -INFINITY, run1 = -INFINITY, acc = 0.f;
  int qn = 0;
  __syncwarp();
  long long t0 = clock64();
  for (int e = 0; e < iters; ++e) {
    const uint8_t *tile = sm + ((e + warp) % NT) * TILE;
    int best0, best1;
    float s0, s1;
    if (V != 1 && V != 4)
      fold_block<G, F>(reinterpret_cast<const uint16_t *>(tile + T * 64), qv, lane, bq, sq, am);
    if (V == 4) {
      uint32_t qe[G][4], qo[G][4];
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          qe[h][i] = bq[(h + i) & 7];
          qo[h][i] = bq[(h + i + 1) & 7];
        }
      block_best_dp4a<G>(tile, qe, qo, lane, best0, best1);
    } else if (V == 2) {
      const uint4 u = *reinterpret_cast<const uint4 *>(tile + lane * 16);
      best0 = static_cast<int>(u.x ^ bq[0]);
      best1 = static_cast<int>(u.y ^ bq[1]);
    } else if (V == 3) {
      best0 = static_cast<int>(bq[0]);
      best1 = static_cast<int>(bq[1]);
    } else {
      block_best<T, F>(tile, bq, T, lane, best0, best1);
    }
    if (V == 3) {
      s0 = __int_as_float(best0 ^ sq);
      s1 = am;
    } else {
      block_scores<F>(best0, best1, sq, am, lane, s0, s1);
    }
    bool keep = false;
    if (gid == 0) {
      run0 = fmaxf(run0, s0);
      run1 = fmaxf(run1, s1);
      keep = s0 >= __fsub_rn(run0, 3.0f) || s1 >= __fsub_rn(run1, 3.0f);
    }
    if (__any_sync(0xffffffffu, keep)) {
      if (lane == 0) {
        qbits[qn & 63] = e;
        __threadfence_block();
      }
      ++qn;
    }
    acc += s0 + s1;
  }
  long long t1 = clock64();
  out[blockIdx.x * blockDim.x + threadIdx.x] = acc + qn;
  if (lane == 0) cyc[blockIdx.x * (blockDim.x / 32) + warp] = t1 - t0;
}

__global__ void sleep_probe(long long *cyc, int ns) {
  long long t0 = clock64();
  for (int i = 0; i < 100; ++i) __nanosleep(ns);
  long long t1 = clock64();
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <int G, int V>
void run(const char *name, int ctas, int warps, const uint8_t *tiles, const uint16_t *q, float *out,
         long long *cyc) {
  const int iters = 2000;
  const size_t smem = NT * TILE + warps * 256;
  cudaFuncSetAttribute(scan_bench<G, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  scan_bench<G, V><<<ctas, warps * 32, smem>>>(tiles, q, 10, out, cyc);
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  cudaEventRecord(a);
  scan_bench<G, V><<<ctas, warps * 32, smem>>>(tiles, q, iters, out, cyc);
  cudaEventRecord(b);
  cudaError_t err = cudaEventSynchronize(b);
  float ms = 0;
  cudaEventElapsedTime(&ms, a, b);
  std::vector<long long> c(ctas * warps);
  cudaMemcpy(c.data(), cyc, c.size() * 8, cudaMemcpyDeviceToHost);
  double mean = 0;
  for (auto v : c) mean += v;
  mean /= c.size();
  printf("%-28s G=%d ctas=%4d warps/cta=%d: %.1f cycles/block/warp, %.3f us/block/warp (event), "
         "blocks/us/SM %.2f  [%s]\n",
         name, G, ctas, warps, mean / iters, ms * 1e3 / iters, (double)ctas * warps * iters / (ms * 1e3) / 148.0,
         cudaGetErrorString(err));
}

int main() {
  const int maxc = 296 * 8;
  uint8_t *tiles;
  uint16_t *q;
  float *out;
  long long *cyc;
  cudaMalloc(&tiles, NT * TILE);
  cudaMalloc(&q, 8 * 128 * 2);
  cudaMalloc(&out, maxc * 32 * 4 * 8);
  cudaMalloc(&cyc, maxc * 8 * 8);
  std::vector<uint8_t> ht(NT * TILE);
  uint32_t x = 12345;
  for (int t = 0; t < NT; ++t) {
    for (int i = 0; i < T * 64; ++i) {
      x = x * 1664525u + 1013904223u;
      ht[t * TILE + i] = (x >> 24) & 0xFF;
    }
    for (int c = 0; c < 128; ++c) {  // scales: bf16 in [0.1, 1]
      x = x * 1664525u + 1013904223u;
      float f = 0.1f + (x >> 8) * (0.9f / 16777216.f);
      uint32_t u;
      memcpy(&u, &f, 4);
      uint16_t h = u >> 16;
      memcpy(&ht[t * TILE + T * 64 + 2 * c], &h, 2);
    }
  }
  std::vector<uint16_t> hq(8 * 128);
  for (auto &v : hq) {
    x = x * 1664525u + 1013904223u;
    float f = ((x >> 8) * (2.f / 16777216.f)) - 1.f;
    uint32_t u;
    memcpy(&u, &f, 4);
    v = u >> 16;
  }
  cudaMemcpy(tiles, ht.data(), ht.size(), cudaMemcpyHostToDevice);
  cudaMemcpy(q, hq.data(), hq.size() * 2, cudaMemcpyHostToDevice);
  for (int w : {1, 2, 4, 8}) {
    run<4, 0>("full (fold+mma+scores)", 1, w, tiles, q, out, cyc);
  }
  run<4, 1>("no fold", 1, 1, tiles, q, out, cyc);
  run<4, 4>("no fold, dp4a scan", 1, 1, tiles, q, out, cyc);
  run<1, 1>("no fold", 1, 1, tiles, q, out, cyc);
  run<1, 4>("no fold, dp4a scan", 1, 1, tiles, q, out, cyc);
  run<8, 1>("no fold", 1, 1, tiles, q, out, cyc);
  run<8, 4>("no fold, dp4a scan", 1, 1, tiles, q, out, cyc);
  run<4, 2>("no mma", 1, 1, tiles, q, out, cyc);
  run<4, 3>("fold only", 1, 1, tiles, q, out, cyc);
  run<1, 0>("full", 1, 1, tiles, q, out, cyc);
  run<8, 0>("full", 1, 1, tiles, q, out, cyc);
  for (int w : {1, 2, 4, 5, 8})
    run<4, 0>("full, 2 CTAs/SM", 296, w, tiles, q, out, cyc);
  run<4, 1>("no fold, 2 CTAs/SM", 296, 4, tiles, q, out, cyc);
  run<4, 2>("no mma, 2 CTAs/SM", 296, 4, tiles, q, out, cyc);
  run<4, 4>("no fold dp4a, 2 CTAs/SM", 296, 4, tiles, q, out, cyc);
  run<4, 4>("no fold dp4a, 2 CTAs/SM", 296, 1, tiles, q, out, cyc);
  run<4, 1>("no fold, 2 CTAs/SM", 296, 1, tiles, q, out, cyc);
  for (int ns : {0, 20, 32, 100, 500}) {
    sleep_probe<<<1, 32>>>(cyc, ns);
    long long c = 0;
    cudaMemcpy(&c, cyc, 8, cudaMemcpyDeviceToHost);
    printf("nanosleep(%d): %.1f cycles per call\n", ns, c / 100.0);
  }
  cudaError_t e = cudaDeviceSynchronize();
  printf("status %s\n", cudaGetErrorString(e));
  return e == cudaSuccess ? 0 : 1;
}
