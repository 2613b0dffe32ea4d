// launch.h -- host-side launchers of the kernels (internal to libzipnn_b200).
#pragma once
#include <cuda_runtime.h>
#include "common.cuh"

namespace zipnn {

// True when the current device is an sm_100 part that can run the kernels (cached per
// device).
bool device_ok();

// Kernel ids of the optional event timing (timing.cu).
enum KernelId { kIdHist = 0, kIdBuild, kIdLayout, kIdEncode, kIdDecode, kIdCodeLengths, kIdPlan, kIdShard, kIdPackHist, kIdPackEncode, kNumKernelIds };

// Brackets one launch with CUDA events on `st` while timing is enabled.
class TimedLaunch {
 public:
  TimedLaunch(int id, cudaStream_t st);
  ~TimedLaunch();
  TimedLaunch(const TimedLaunch&) = delete;
  TimedLaunch& operator=(const TimedLaunch&) = delete;

 private:
  int id_;
  cudaStream_t st_;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

// Histograms. With ws (compress), also every tile's counts (and FP32's zero-run bitmaps);
// the chunks' codes follow in launch_build_chunks.
cudaError_t launch_split_hist(const void* src, const Geo& g, uint32_t* hist, uint32_t* nonzero, const Ws* ws,
                              const PlanDev& plan, cudaStream_t st);
// Compress: the chunks' codes and tile offsets, after launch_split_hist (one block per chunk).
cudaError_t launch_build_chunks(const Geo& g, const Ws& ws, const PlanDev& plan, cudaStream_t st);
cudaError_t launch_code_lengths(const uint64_t* hist, uint32_t count, uint32_t alphabet_size, uint8_t* lens,
                                uint32_t* enc, cudaStream_t st);
cudaError_t launch_layout(const Geo& g, const Ws& ws, const PlanDev& plan, uint8_t* out, cudaStream_t st);
uint32_t layout_tiles(uint32_t n_entries);
// BF16 encode: persistent blocks, tile bit offsets from the per-tile histograms.
cudaError_t launch_encode_bf16(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st);
// FP32 encode: the same scheme with three byte planes.
cudaError_t launch_encode_fp32(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st);
// FP8 and FP4 encode: the same scheme, with grouped code tables and bit-parallel packing.
cudaError_t launch_encode_sub(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st);
// Packed exponents (pack.cu): the plan's list, the chunks' pair counts, the groups' sums,
// and the PACK payloads.
cudaError_t launch_pack_select(const uint32_t* hist, uint32_t C, uint32_t NE, uint32_t max_pack, uint8_t* exps,
                               uint32_t* k_out, cudaStream_t st);
cudaError_t launch_pack_hist(const void* src, const Geo& g, const Ws& ws, const PlanDev& plan, cudaStream_t st);
cudaError_t launch_pack_group_sums(const uint32_t* pack_hist, const uint32_t* assign, uint32_t C, uint64_t* gsum,
                                   cudaStream_t st);
cudaError_t launch_encode_pack(const void* src, const Geo& g, const Ws& ws, const PlanDev& plan, uint8_t* out,
                               cudaStream_t st);
cudaError_t launch_decode(const uint8_t* in, uint64_t in_bytes, const Geo& g, uint8_t* out, uint32_t* status,
                          cudaStream_t st);
// One tensor of a batched decode (device table); chunk0 = its first chunk in the batch.
struct DecodeItem {
  const uint8_t* in;
  uint64_t in_bytes;
  uint64_t n;
  uint8_t* out;
  uint64_t chunk0;
};
// All chunks of `count` tensors of one dtype and chunk size in one launch; g carries the
// dtype, chunk_bytes and m0 (n and n_chunks come from each item).
cudaError_t launch_decode_batch(const DecodeItem* items, uint32_t count, const Geo& g, uint32_t total_chunks,
                                uint32_t* status, cudaStream_t st);

// plan (grouping) steps
struct KmeansDev {
  const uint32_t* hist;  // [C][n_entropy][256] (entropy stream 0 is the feature)
  uint32_t C, A, NE, G;
  uint64_t m0, n;
  double* mu;            // [G][A]
  uint32_t* assign;      // [C]
  uint32_t* perm;        // [C]
  uint32_t* changed;     // [1]
  uint64_t* gsum;        // [NE][G][256]
};
cudaError_t launch_kmeans_init(const KmeansDev& k, uint64_t seed, cudaStream_t st);
cudaError_t launch_kmeans_assign(const KmeansDev& k, cudaStream_t st);
cudaError_t launch_kmeans_update(const KmeansDev& k, cudaStream_t st);
cudaError_t launch_group_sums(const KmeansDev& k, cudaStream_t st);
cudaError_t launch_canonical(const uint8_t* lens, uint32_t count, uint32_t* enc, cudaStream_t st);
cudaError_t launch_identity_assign(uint32_t* assign, uint32_t C, cudaStream_t st);

}  // namespace zipnn
