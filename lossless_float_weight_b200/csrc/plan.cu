// plan.cu -- the reusable shared-code setup ("NeuralZip: Reusable Setup for Fast
// Lossless Compression", abstract: chunks with similar exponent distributions are
// grouped and share one Huffman code; the setup is computed once and reused).
//
// The grouping is Lloyd's k-means over the normalised exponent histograms
// x_c[i] = h_c[i] / m_c, seeded by a partial Fisher-Yates shuffle driven by SplitMix64
// (Steele, Lea and Flood, 2014). Every double operation is a separately rounded IEEE
// operation (__dsub_rn, __dmul_rn, __dadd_rn, __ddiv_rn) in a fixed order, so the
// result does not depend on the launch shape.
#include "common.cuh"
#include "huffman.cuh"
#include "launch.h"

namespace zipnn {

__device__ __forceinline__ uint64_t splitmix64(uint64_t& state) {
  uint64_t z = (state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double feature(const KmeansDev& k, uint32_t c, uint32_t i) {
  const uint64_t lo = (uint64_t)c * k.m0;
  const uint64_t m = k.n - lo < k.m0 ? k.n - lo : k.m0;
  return __ddiv_rn((double)k.hist[((uint64_t)c * k.NE) * 256 + i], (double)m);
}

__global__ void k_km_init(KmeansDev k, uint64_t seed) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  uint64_t state = seed;
  for (uint32_t j = 0; j < k.G; j++) {
    const uint64_t r = j + splitmix64(state) % (uint64_t)(k.C - j);
    const uint32_t t = k.perm[j];
    k.perm[j] = k.perm[r];
    k.perm[r] = t;
    for (uint32_t i = 0; i < k.A; i++) k.mu[(uint64_t)j * k.A + i] = feature(k, k.perm[j], i);
  }
}

__global__ void k_iota(uint32_t* p, uint32_t n, uint32_t fill_assign, uint32_t* assign) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    p[i] = i;
    assign[i] = fill_assign;
  }
}

// nearest centre of every chunk (squared distance summed over i ascending; ties to the
// smaller group)
__global__ void k_km_assign(KmeansDev k) {
  const uint32_t c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= k.C) return;
  uint32_t best = 0;
  double bd = 0.0;
  for (uint32_t j = 0; j < k.G; j++) {
    double s = 0.0;
    for (uint32_t i = 0; i < k.A; i++) {
      const double t = __dsub_rn(feature(k, c, i), k.mu[(uint64_t)j * k.A + i]);
      s = __dadd_rn(s, __dmul_rn(t, t));
    }
    if (j == 0 || s < bd) {
      bd = s;
      best = j;
    }
  }
  if (k.assign[c] != best) {
    k.assign[c] = best;
    *k.changed = 1u;
  }
}

// centre j, coordinate i: mean of the members, summed in ascending chunk order; an
// empty group keeps its centre
__global__ void k_km_update(KmeansDev k) {
  const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= k.G * k.A) return;
  const uint32_t j = t / k.A, i = t % k.A;
  double s = 0.0;
  uint64_t members = 0;
  for (uint32_t c = 0; c < k.C; c++)
    if (k.assign[c] == j) {
      s = __dadd_rn(s, feature(k, c, i));
      members++;
    }
  if (members) k.mu[(uint64_t)j * k.A + i] = __ddiv_rn(s, (double)members);
}

// summed histograms of each group, per entropy stream
__global__ void k_group_sums(KmeansDev k) {
  const uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (uint64_t)k.C * k.NE * 256) return;
  const uint32_t c = (uint32_t)(t / (k.NE * 256));
  const uint32_t r = (uint32_t)(t % (k.NE * 256));
  const uint32_t e = r / 256, sym = r % 256;
  const uint32_t v = k.hist[t];
  if (v) atomicAdd(reinterpret_cast<unsigned long long*>(k.gsum + ((uint64_t)e * k.G + k.assign[c]) * 256 + sym),
                   (unsigned long long)v);
}

// canonical code values for imported length records (one warp per record)
__global__ void k_canonical(const uint8_t* lens, uint32_t count, uint32_t* enc) {
  const uint32_t r = blockIdx.x;
  if (r < count && threadIdx.x < 32) warp_canonical(lens + (uint64_t)r * 256, enc + (uint64_t)r * 256);
}

cudaError_t launch_kmeans_init(const KmeansDev& k, uint64_t seed, cudaStream_t st) {
  k_iota<<<(k.C + 255) / 256, 256, 0, st>>>(k.perm, k.C, 0xFFFFFFFFu, k.assign);
  k_km_init<<<1, 32, 0, st>>>(k, seed);
  return cudaGetLastError();
}

cudaError_t launch_kmeans_assign(const KmeansDev& k, cudaStream_t st) {
  k_km_assign<<<(k.C + 127) / 128, 128, 0, st>>>(k);
  return cudaGetLastError();
}

cudaError_t launch_kmeans_update(const KmeansDev& k, cudaStream_t st) {
  k_km_update<<<(k.G * k.A + 127) / 128, 128, 0, st>>>(k);
  return cudaGetLastError();
}

cudaError_t launch_group_sums(const KmeansDev& k, cudaStream_t st) {
  const uint64_t n = (uint64_t)k.C * k.NE * 256;
  k_group_sums<<<(uint32_t)((n + 255) / 256), 256, 0, st>>>(k);
  return cudaGetLastError();
}

cudaError_t launch_canonical(const uint8_t* lens, uint32_t count, uint32_t* enc, cudaStream_t st) {
  if (!count) return cudaSuccess;
  k_canonical<<<count, 32, 0, st>>>(lens, count, enc);
  return cudaGetLastError();
}

// chunk c is group c when there are no more chunks than groups
__global__ void k_identity_assign(uint32_t* assign, uint32_t C) {
  const uint32_t c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < C) assign[c] = c;
}

cudaError_t launch_identity_assign(uint32_t* assign, uint32_t C, cudaStream_t st) {
  k_identity_assign<<<(C + 255) / 256, 256, 0, st>>>(assign, C);
  return cudaGetLastError();
}

}  // namespace zipnn
