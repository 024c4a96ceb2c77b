// stepq_internal.h -- pool object and kernel launchers shared by the C ABI and the kernels.
#pragma once

#include <cstdint>
#include <vector>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "stepq.h"

struct stepq_pool {
    int32_t num_slots = 0, H = 0, Hk = 0, gate_mode = 0, in_dtype = 0;
    std::vector<uint8_t> bits;          // [H]
    std::vector<long long> offs;        // [H] byte offset of each head block in a slot
    long long slot_stride = 0;          // bytes per slot
    long long total = 0;                // bytes of the pool
    int max_block = 0;                  // largest quantized head block (bytes)
    int npiv = 0;                       // FP16 pivot heads (width 16), visited after the others
    int device = 0;
    int num_sms = 0;
    int32_t debug = 0;                  // STEPQ_DEBUG_* flags (stepq_pool_set_debug)
    uint8_t *d_pool = nullptr;          // [num_slots * slot_stride]
    long long *d_offs = nullptr;        // [H]
    uint8_t *d_bits = nullptr;          // [H]
    int32_t *d_order = nullptr;         // [H] head processing order (widths 4, 6, 8, then pivots)
    int *d_flag = nullptr;              // sticky device flag (STEPQ_FLAG_* bits)
    float *d_impact = nullptr;          // [H, d_k] normalized row-impact weights (impact fit), or null
    // heads with per-key-row widths (width 0 in bits): rows of width 8 and 4, padded panel
    // bytes, block bytes, stored row -> key row; null when the pool has none
    std::vector<uint8_t> rn8, rn4;      // [H]
    std::vector<int32_t> rpb;           // [H]
    std::vector<uint8_t> perm;          // [H * d_k]
    int32_t *d_blk = nullptr;           // [H] block bytes of every head
    uint8_t *d_rn8 = nullptr, *d_rn4 = nullptr, *d_perm = nullptr;
    int32_t *d_rpb = nullptr;
    int decode_grid = 0;                // persistent CTAs for the decode kernel
    size_t decode_smem = 0;             // dynamic shared memory of the decode kernel
    int stage_bytes = 0;
    int blk_cap = 0;
    // pools with FP16 pivot heads: the pivot kernel's stream, forked from and joined back to
    // the caller's stream in every step (the two kernels share no data)
    cudaStream_t s_piv = nullptr;
    cudaEvent_t ev_pfork = nullptr, ev_pjoin = nullptr;
    // host-buffer decode (stepq_decode_step_host): two device staging buffers used in turn,
    // the copy-in and copy-out streams, and the events that chain copy-in -> step -> copy-out;
    // created on first use
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_step[2] = {nullptr, nullptr}, ev_out[2] = {nullptr, nullptr};
    uint8_t *d_host_stage[2] = {nullptr, nullptr};
    size_t host_stage_cap = 0;          // bytes of each staging buffer
    long long host_calls = 0;
};

namespace stepq {

constexpr int kMaxHeads = 256;

// NVTX range over the host side of a data-path call (argument checks and the enqueue of its
// copies and kernels).  A profiler that records NVTX attributes the kernels the call launches
// to the range, e.g. ncu --nvtx --nvtx-include "stepq_decode_step/"; with no tool attached a
// push and a pop cost a few nanoseconds.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Launchers (return a cudaError_t from the launch).
cudaError_t decode_configure(stepq_pool *p);
cudaError_t launch_decode(const stepq_pool *p, const int32_t *slot_ids, int n, const void *q,
                          const void *k, const void *v, const void *alpha, const void *beta,
                          float *y, cudaStream_t stream);
cudaError_t launch_wait_check(int *flag, cudaStream_t stream);
cudaError_t launch_load_fp32(const stepq_pool *p, const int32_t *slot_ids, int n, const float *S,
                             cudaStream_t stream);
cudaError_t launch_dump_fp32(const stepq_pool *p, const int32_t *slot_ids, int n, float *S,
                             cudaStream_t stream);
cudaError_t launch_copy_slots(const stepq_pool *p, const int32_t *slot_ids, int n, const uint8_t *src,
                              uint8_t *dst, bool into_pool, cudaStream_t stream);

}  // namespace stepq
