// stepq_capi.cu -- the C ABI of libstepq (declared in include/stepq.h): pool
// management, argument validation and kernel launches.  Every step of the decode
// path runs in the kernels of stepq_decode.cu and stepq_io.cu; this file only checks
// arguments and launches.
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "stepq_internal.h"
#include "stepq_tile.cuh"

using stepq::block_bytes;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int status_of(cudaError_t e)
{
    if (e == cudaSuccess) return STEPQ_OK;
    if (e == cudaErrorMemoryAllocation) return STEPQ_OUT_OF_MEMORY;
    return STEPQ_CUDA_ERROR;
}

// The pool's device must be current for every call that touches it.
int check_device(const stepq_pool *p)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return STEPQ_CUDA_ERROR;
    return dev == p->device ? STEPQ_OK : STEPQ_INVALID_ARG;
}

int check_slots(const stepq_pool *p, const int32_t *slot_ids, int32_t n)
{
    if (!p || n < 0) return STEPQ_INVALID_ARG;
    if (n > 0 && (!slot_ids || !aligned_to(slot_ids, 4))) return STEPQ_INVALID_ARG;
    if (n > p->num_slots || n > 65535) return STEPQ_INVALID_ARG;
    return check_device(p);
}

// Distinct ids in [0, num_slots) (host array).
int host_check_slot_ids(const int32_t *ids, int32_t n, int32_t num_slots)
{
    if (n < 0 || num_slots <= 0 || (n > 0 && !ids)) return STEPQ_INVALID_ARG;
    std::vector<uint8_t> seen;
    try {
        seen.assign(size_t(num_slots), 0);
    } catch (...) {
        return STEPQ_OUT_OF_MEMORY;
    }
    for (int32_t i = 0; i < n; ++i) {
        const int32_t s = ids[i];
        if (s < 0 || s >= num_slots || seen[size_t(s)]) return STEPQ_INVALID_ARG;
        seen[size_t(s)] = 1;
    }
    return STEPQ_OK;
}

// Debug mode (STEPQ_DEBUG_SLOTS): copy a call's device slot ids to the host and check them
// before any device work of the call (synchronizes `stream`).
int debug_check_slots(const stepq_pool *p, const int32_t *slot_ids, int32_t n, cudaStream_t stream)
{
    if (!(p->debug & STEPQ_DEBUG_SLOTS) || n == 0) return STEPQ_OK;
    std::vector<int32_t> h;
    try {
        h.resize(size_t(n));
    } catch (...) {
        return STEPQ_OUT_OF_MEMORY;
    }
    cudaError_t e = cudaMemcpyAsync(h.data(), slot_ids, sizeof(int32_t) * size_t(n), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return status_of(e);
    return host_check_slot_ids(h.data(), n, p->num_slots);
}

void free_pool(stepq_pool *p)
{
    if (!p) return;
    cudaFree(p->d_pool);
    cudaFree(p->d_offs);
    cudaFree(p->d_bits);
    cudaFree(p->d_order);
    cudaFree(p->d_flag);
    cudaFree(p->d_impact);
    cudaFree(p->d_blk);
    cudaFree(p->d_rn8);
    cudaFree(p->d_rn4);
    cudaFree(p->d_rpb);
    cudaFree(p->d_perm);
    for (int b = 0; b < 2; ++b) {
        cudaFree(p->d_host_stage[b]);
        if (p->ev_in[b]) cudaEventDestroy(p->ev_in[b]);
        if (p->ev_step[b]) cudaEventDestroy(p->ev_step[b]);
        if (p->ev_out[b]) cudaEventDestroy(p->ev_out[b]);
    }
    if (p->ev_pfork) cudaEventDestroy(p->ev_pfork);
    if (p->ev_pjoin) cudaEventDestroy(p->ev_pjoin);
    if (p->s_piv) cudaStreamDestroy(p->s_piv);
    if (p->s_in) cudaStreamDestroy(p->s_in);
    if (p->s_out) cudaStreamDestroy(p->s_out);
    delete p;
}

// ---- host-buffer decode: byte offsets of one call's inputs and output in a staging buffer
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct HostLayout {
    size_t slots, q, k, v, alpha, beta, y, total;
    size_t qk_bytes, v_bytes, alpha_bytes, beta_bytes, y_bytes;
};

HostLayout host_layout(const stepq_pool *p, int n)
{
    const size_t esz = p->in_dtype == STEPQ_DTYPE_BF16 ? 2 : 4;
    HostLayout L;
    L.qk_bytes = size_t(n) * p->Hk * 128 * esz;
    L.v_bytes = size_t(n) * p->H * 128 * esz;
    L.alpha_bytes = size_t(n) * p->H * (p->gate_mode == STEPQ_GATE_KDA ? 128 : 1) * esz;
    L.beta_bytes = size_t(n) * p->H * esz;
    L.y_bytes = size_t(n) * p->H * 128 * 4;
    size_t o = 0;
    L.slots = o; o += round256(size_t(n) * 4);
    L.q = o; o += round256(L.qk_bytes);
    L.k = o; o += round256(L.qk_bytes);
    L.v = o; o += round256(L.v_bytes);
    L.alpha = o; o += round256(L.alpha_bytes);
    L.beta = o; o += round256(L.beta_bytes);
    L.y = o; o += round256(L.y_bytes);
    L.total = o;
    return L;
}

// Streams, events and staging buffers of the host-buffer path: created on the first call,
// regrown (once every earlier use has finished) when a call needs more room.
int host_prepare(stepq_pool *p, size_t bytes)
{
    cudaError_t e = cudaSuccess;
    if (!p->s_in) {
        e = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking);
        for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
            e = cudaEventCreateWithFlags(&p->ev_in[b], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ev_step[b], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ev_out[b], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) return status_of(e);
    }
    if (bytes <= p->host_stage_cap) return STEPQ_OK;
    // every earlier use of a staging buffer ends with its copy-out
    for (int b = 0; b < 2 && e == cudaSuccess; ++b) e = cudaEventSynchronize(p->ev_out[b]);
    if (e != cudaSuccess) return status_of(e);
    for (int b = 0; b < 2; ++b) {
        cudaFree(p->d_host_stage[b]);
        p->d_host_stage[b] = nullptr;
    }
    p->host_stage_cap = 0;
    for (int b = 0; b < 2; ++b) {
        e = cudaMalloc(&p->d_host_stage[b], bytes);
        if (e != cudaSuccess) return status_of(e);
    }
    p->host_stage_cap = bytes;
    return STEPQ_OK;
}

}  // namespace

extern "C" {

const char *stepq_status_string(int status)
{
    switch (status) {
    case STEPQ_OK: return "ok";
    case STEPQ_INVALID_ARG: return "invalid argument";
    case STEPQ_OUT_OF_MEMORY: return "out of memory";
    case STEPQ_CUDA_ERROR: return "CUDA error";
    case STEPQ_UNSUPPORTED: return "unsupported configuration (d_k = d_v = 128, bits in {4, 6, 8, 16}, row bits in {4, 6, 8})";
    case STEPQ_DEVICE_FLAG: return "device flag set (bad slot id or kernel wait timeout)";
    default: return "unknown status";
    }
}

}  // extern "C"

namespace {

// Pool creation; row_bits (host [H, d_k] or null) gives the per-key-row widths of the heads of
// width 0.
int create_pool(const stepq_pool_desc *desc, const uint8_t *row_bits, stepq_pool **out)
{
    if (!desc || !out || !desc->head_bits) return STEPQ_INVALID_ARG;
    *out = nullptr;
    if (desc->num_slots <= 0 || desc->num_heads <= 0 || desc->num_key_heads <= 0) return STEPQ_INVALID_ARG;
    if (desc->num_heads % desc->num_key_heads != 0) return STEPQ_INVALID_ARG;
    if (desc->num_heads > stepq::kMaxHeads) return STEPQ_UNSUPPORTED;
    if (desc->gate_mode != STEPQ_GATE_GDN && desc->gate_mode != STEPQ_GATE_KDA) return STEPQ_INVALID_ARG;
    if (desc->in_dtype != STEPQ_DTYPE_F32 && desc->in_dtype != STEPQ_DTYPE_BF16) return STEPQ_INVALID_ARG;
    if (desc->d_k != stepq::DK || desc->d_v != stepq::DV) return STEPQ_UNSUPPORTED;
    bool any_rows = false;
    for (int h = 0; h < desc->num_heads; ++h) {
        const int b = desc->head_bits[h];
        if (b == 0 && row_bits) {
            any_rows = true;
            for (int i = 0; i < stepq::DK; ++i) {
                const int rb = row_bits[h * stepq::DK + i];
                if (rb != 4 && rb != 6 && rb != 8) return STEPQ_UNSUPPORTED;
            }
        } else if (b != 4 && b != 6 && b != 8 && b != 16) {
            return STEPQ_UNSUPPORTED;
        }
    }
    stepq_pool *p = new (std::nothrow) stepq_pool();
    if (!p) return STEPQ_OUT_OF_MEMORY;
    p->num_slots = desc->num_slots;
    p->H = desc->num_heads;
    p->Hk = desc->num_key_heads;
    p->gate_mode = desc->gate_mode;
    p->in_dtype = desc->in_dtype;
    p->bits.assign(desc->head_bits, desc->head_bits + p->H);
    p->offs.resize(p->H);
    std::vector<int32_t> blk(p->H);
    if (any_rows) {
        p->rn8.assign(p->H, 0);
        p->rn4.assign(p->H, 0);
        p->rpb.assign(p->H, 0);
        p->perm.assign(size_t(p->H) * stepq::DK, 0);
    }
    long long off = 0;
    for (int h = 0; h < p->H; ++h) {
        p->offs[h] = off;
        if (p->bits[h] == 0) {
            // rows stored 8-bit, then 4-bit, then 6-bit (ascending key row in each group);
            // panels padded to 16 bytes
            const uint8_t *rb = row_bits + h * stepq::DK;
            int n[3] = {0, 0, 0}, pos = 0;
            const int widths[3] = {8, 4, 6};
            for (int wdt = 0; wdt < 3; ++wdt)
                for (int i = 0; i < stepq::DK; ++i)
                    if (rb[i] == widths[wdt]) {
                        p->perm[size_t(h) * stepq::DK + pos++] = uint8_t(i);
                        ++n[wdt];
                    }
            p->rn8[h] = uint8_t(n[0]);
            p->rn4[h] = uint8_t(n[1]);
            p->rpb[h] = (16 * n[0] + 8 * n[1] + 12 * n[2] + 15) / 16 * 16;
            blk[h] = stepq::NPANEL * p->rpb[h] + 4 * stepq::DK + 4 * stepq::DV;
        } else {
            blk[h] = block_bytes(p->bits[h]);
        }
        off += blk[h];
        if (p->bits[h] == 16)
            ++p->npiv;
        else if (blk[h] > p->max_block)
            p->max_block = blk[h];
    }
    p->slot_stride = off;
    p->total = off * (long long)p->num_slots;
    cudaError_t e = cudaGetDevice(&p->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_pool, size_t(p->total));
    if (e == cudaSuccess) e = cudaMalloc(&p->d_offs, sizeof(long long) * p->H);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_bits, size_t(p->H));
    if (e == cudaSuccess) e = cudaMalloc(&p->d_order, sizeof(int32_t) * p->H);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_flag, sizeof(int));
    if (e == cudaSuccess && p->npiv > 0) {
        e = cudaStreamCreateWithFlags(&p->s_piv, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ev_pfork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ev_pjoin, cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaMemset(p->d_pool, 0, size_t(p->total));
    if (e == cudaSuccess) e = cudaMemset(p->d_flag, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaMemcpy(p->d_offs, p->offs.data(), sizeof(long long) * p->H, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(p->d_bits, p->bits.data(), size_t(p->H), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && any_rows) {
        e = cudaMalloc(&p->d_blk, sizeof(int32_t) * p->H);
        if (e == cudaSuccess) e = cudaMalloc(&p->d_rn8, size_t(p->H));
        if (e == cudaSuccess) e = cudaMalloc(&p->d_rn4, size_t(p->H));
        if (e == cudaSuccess) e = cudaMalloc(&p->d_rpb, sizeof(int32_t) * p->H);
        if (e == cudaSuccess) e = cudaMalloc(&p->d_perm, p->perm.size());
        if (e == cudaSuccess) e = cudaMemcpy(p->d_blk, blk.data(), sizeof(int32_t) * p->H, cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = cudaMemcpy(p->d_rn8, p->rn8.data(), size_t(p->H), cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = cudaMemcpy(p->d_rn4, p->rn4.data(), size_t(p->H), cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = cudaMemcpy(p->d_rpb, p->rpb.data(), sizeof(int32_t) * p->H, cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = cudaMemcpy(p->d_perm, p->perm.data(), p->perm.size(), cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess) {
        // the decode kernel visits heads grouped by bit width (stable within a width): 4, 6,
        // 8, per-key-row widths; the FP16 pivot heads come last and go to their own kernel
        std::vector<int32_t> order;
        for (int w : {4, 6, 8, 0, 16})
            for (int h = 0; h < p->H; ++h)
                if (p->bits[h] == w) order.push_back(h);
        e = cudaMemcpy(p->d_order, order.data(), sizeof(int32_t) * p->H, cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess) e = stepq::decode_configure(p);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        free_pool(p);
        return status_of(e);
    }
    *out = p;
    return STEPQ_OK;
}

}  // namespace

extern "C" {

int stepq_pool_create(const stepq_pool_desc *desc, stepq_pool **out) { return create_pool(desc, nullptr, out); }

int stepq_pool_create_rows(const stepq_pool_desc *desc, const uint8_t *row_bits, stepq_pool **out)
{
    if (!row_bits) return STEPQ_INVALID_ARG;
    return create_pool(desc, row_bits, out);
}

int stepq_pool_destroy(stepq_pool *pool)
{
    if (!pool) return STEPQ_OK;
    const cudaError_t e = cudaDeviceSynchronize();
    free_pool(pool);
    return status_of(e);
}

int stepq_pool_bytes(const stepq_pool *pool, size_t *slot_stride, size_t *total)
{
    if (!pool) return STEPQ_INVALID_ARG;
    if (slot_stride) *slot_stride = size_t(pool->slot_stride);
    if (total) *total = size_t(pool->total);
    return STEPQ_OK;
}

int stepq_pool_head_offset(const stepq_pool *pool, int32_t h, size_t *offset)
{
    if (!pool || !offset || h < 0 || h >= pool->H) return STEPQ_INVALID_ARG;
    *offset = size_t(pool->offs[h]);
    return STEPQ_OK;
}

int stepq_pool_load_fp32(stepq_pool *pool, const int32_t *slot_ids, int32_t n, const float *S,
                         stepq_stream stream)
{
    const stepq::NvtxRange range("stepq_pool_load_fp32");
    int st = check_slots(pool, slot_ids, n);
    if (st != STEPQ_OK) return st;
    if (n == 0) return STEPQ_OK;
    if (!S || !aligned16(S)) return STEPQ_INVALID_ARG;
    st = debug_check_slots(pool, slot_ids, n, stream);
    if (st != STEPQ_OK) return st;
    return status_of(stepq::launch_load_fp32(pool, slot_ids, n, S, stream));
}

int stepq_pool_load_packed(stepq_pool *pool, const int32_t *slot_ids, int32_t n, const uint8_t *bytes,
                           stepq_stream stream)
{
    const stepq::NvtxRange range("stepq_pool_load_packed");
    int st = check_slots(pool, slot_ids, n);
    if (st != STEPQ_OK) return st;
    if (n == 0) return STEPQ_OK;
    if (!bytes || !aligned16(bytes)) return STEPQ_INVALID_ARG;
    st = debug_check_slots(pool, slot_ids, n, stream);
    if (st != STEPQ_OK) return st;
    return status_of(stepq::launch_copy_slots(pool, slot_ids, n, bytes, nullptr, true, stream));
}

int stepq_pool_dump_fp32(const stepq_pool *pool, const int32_t *slot_ids, int32_t n, float *S_out,
                         stepq_stream stream)
{
    const stepq::NvtxRange range("stepq_pool_dump_fp32");
    int st = check_slots(pool, slot_ids, n);
    if (st != STEPQ_OK) return st;
    if (n == 0) return STEPQ_OK;
    if (!S_out || !aligned16(S_out)) return STEPQ_INVALID_ARG;
    st = debug_check_slots(pool, slot_ids, n, stream);
    if (st != STEPQ_OK) return st;
    return status_of(stepq::launch_dump_fp32(pool, slot_ids, n, S_out, stream));
}

int stepq_pool_dump_packed(const stepq_pool *pool, const int32_t *slot_ids, int32_t n, uint8_t *bytes_out,
                           stepq_stream stream)
{
    const stepq::NvtxRange range("stepq_pool_dump_packed");
    int st = check_slots(pool, slot_ids, n);
    if (st != STEPQ_OK) return st;
    if (n == 0) return STEPQ_OK;
    if (!bytes_out || !aligned16(bytes_out)) return STEPQ_INVALID_ARG;
    st = debug_check_slots(pool, slot_ids, n, stream);
    if (st != STEPQ_OK) return st;
    return status_of(stepq::launch_copy_slots(pool, slot_ids, n, nullptr, bytes_out, false, stream));
}

int stepq_decode_step(stepq_pool *pool, const int32_t *slot_ids, int32_t n, const void *q, const void *k,
                      const void *v, const void *alpha, const void *beta, float *y, stepq_stream stream)
{
    const stepq::NvtxRange range("stepq_decode_step");
    int st = check_slots(pool, slot_ids, n);
    if (st != STEPQ_OK) return st;
    if (n == 0) return STEPQ_OK;
    if (!q || !k || !v || !alpha || !beta || !y) return STEPQ_INVALID_ARG;
    // q, k, v (and the KDA gate) are bulk-copied: 16-byte aligned rows
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned_to(y, 4)) return STEPQ_INVALID_ARG;
    const size_t esz = pool->in_dtype == STEPQ_DTYPE_BF16 ? 2 : 4;
    if (pool->gate_mode == STEPQ_GATE_KDA ? !aligned16(alpha) : !aligned_to(alpha, esz)) return STEPQ_INVALID_ARG;
    if (!aligned_to(beta, esz)) return STEPQ_INVALID_ARG;
    st = debug_check_slots(pool, slot_ids, n, stream);
    if (st != STEPQ_OK) return st;
    return status_of(stepq::launch_decode(pool, slot_ids, n, q, k, v, alpha, beta, y, stream));
}

int stepq_decode_step_host(stepq_pool *pool, const int32_t *slot_ids, int32_t n, const void *q, const void *k,
                           const void *v, const void *alpha, const void *beta, float *y, stepq_stream stream)
{
    const stepq::NvtxRange range("stepq_decode_step_host");
    if (!pool || n < 0 || n > pool->num_slots || n > 65535) return STEPQ_INVALID_ARG;
    int st = check_device(pool);
    if (st != STEPQ_OK) return st;
    if (n == 0) return STEPQ_OK;
    if (!slot_ids || !q || !k || !v || !alpha || !beta || !y) return STEPQ_INVALID_ARG;
    if (pool->debug & STEPQ_DEBUG_SLOTS) {
        st = host_check_slot_ids(slot_ids, n, pool->num_slots);
        if (st != STEPQ_OK) return st;
    }
    const HostLayout L = host_layout(pool, n);
    st = host_prepare(pool, L.total);
    if (st != STEPQ_OK) return st;
    const int b = int(pool->host_calls & 1);
    uint8_t *d = pool->d_host_stage[b];
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice;
    // inputs laid out as one contiguous image (stepq_host_image_layout) go in one copy
    const uint8_t *img = reinterpret_cast<const uint8_t *>(slot_ids);
    const bool one_image = q == img + L.q && k == img + L.k && v == img + L.v && alpha == img + L.alpha &&
                           beta == img + L.beta;
    // copy-in, once the step that last read this staging buffer is done
    cudaError_t e = cudaStreamWaitEvent(pool->s_in, pool->ev_step[b], 0);
    if (one_image) {
        if (e == cudaSuccess) e = cudaMemcpyAsync(d, img, L.beta + L.beta_bytes, h2d, pool->s_in);
    } else {
        if (e == cudaSuccess) e = cudaMemcpyAsync(d + L.slots, slot_ids, size_t(n) * 4, h2d, pool->s_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(d + L.q, q, L.qk_bytes, h2d, pool->s_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(d + L.k, k, L.qk_bytes, h2d, pool->s_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(d + L.v, v, L.v_bytes, h2d, pool->s_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(d + L.alpha, alpha, L.alpha_bytes, h2d, pool->s_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(d + L.beta, beta, L.beta_bytes, h2d, pool->s_in);
    }
    if (e == cudaSuccess) e = cudaEventRecord(pool->ev_in[b], pool->s_in);
    // the step on the caller's stream, once its inputs are in and the copy-out that last read
    // this buffer's y is done
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, pool->ev_in[b], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, pool->ev_out[b], 0);
    if (e == cudaSuccess)
        e = stepq::launch_decode(pool, reinterpret_cast<const int32_t *>(d + L.slots), n, d + L.q, d + L.k, d + L.v,
                                 d + L.alpha, d + L.beta, reinterpret_cast<float *>(d + L.y), stream);
    if (e == cudaSuccess) e = cudaEventRecord(pool->ev_step[b], stream);
    // copy-out of y
    if (e == cudaSuccess) e = cudaStreamWaitEvent(pool->s_out, pool->ev_step[b], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(y, d + L.y, L.y_bytes, cudaMemcpyDeviceToHost, pool->s_out);
    if (e == cudaSuccess) e = cudaEventRecord(pool->ev_out[b], pool->s_out);
    ++pool->host_calls;
    return status_of(e);
}

int stepq_host_image_layout(const stepq_pool *pool, int32_t n, size_t *offsets_out, size_t *total_out)
{
    if (!pool || !offsets_out || n < 0 || n > pool->num_slots || n > 65535) return STEPQ_INVALID_ARG;
    const HostLayout L = host_layout(pool, n);
    const size_t o[6] = {L.slots, L.q, L.k, L.v, L.alpha, L.beta};
    for (int i = 0; i < 6; ++i) offsets_out[i] = o[i];
    if (total_out) *total_out = L.beta + L.beta_bytes;
    return STEPQ_OK;
}

int stepq_pool_host_wait(stepq_pool *pool, stepq_stream stream)
{
    if (!pool) return STEPQ_INVALID_ARG;
    int st = check_device(pool);
    if (st != STEPQ_OK || !pool->s_in) return st;
    cudaError_t e = cudaSuccess;
    for (int b = 0; b < 2 && e == cudaSuccess; ++b) e = cudaStreamWaitEvent(stream, pool->ev_out[b], 0);
    return status_of(e);
}

int stepq_pool_set_impact(stepq_pool *pool, const float *impact)
{
    if (!pool) return STEPQ_INVALID_ARG;
    int st = check_device(pool);
    if (st != STEPQ_OK) return st;
    cudaError_t e = cudaDeviceSynchronize();           // no launch in flight reads the table
    if (e != cudaSuccess) return status_of(e);
    if (!impact) {
        e = cudaFree(pool->d_impact);
        pool->d_impact = nullptr;
        return status_of(e);
    }
    const int n = pool->H * stepq::DK;
    std::vector<float> w(size_t(n), 0.0f);
    for (int h = 0; h < pool->H; ++h) {
        double sum = 0.0;
        for (int i = 0; i < stepq::DK; ++i) {
            const float o = impact[h * stepq::DK + i];
            if (!(o > 0.0f) || !(o < 3.0e38f)) return STEPQ_INVALID_ARG;     // positive and finite
            sum += double(o);
        }
        for (int i = 0; i < stepq::DK; ++i)
            w[size_t(h) * stepq::DK + i] = float(double(impact[h * stepq::DK + i]) / (sum / stepq::DK));
    }
    if (!pool->d_impact) {
        e = cudaMalloc(&pool->d_impact, sizeof(float) * size_t(n));
        if (e != cudaSuccess) return status_of(e);
    }
    e = cudaMemcpy(pool->d_impact, w.data(), sizeof(float) * size_t(n), cudaMemcpyHostToDevice);
    return status_of(e);
}

int stepq_pool_set_debug(stepq_pool *pool, int32_t flags)
{
    if (!pool || (flags & ~int32_t(STEPQ_DEBUG_SLOTS)) != 0) return STEPQ_INVALID_ARG;
    pool->debug = flags;
    return STEPQ_OK;
}

int stepq_check_slot_ids(const int32_t *slot_ids, int32_t n, int32_t num_slots)
{
    return host_check_slot_ids(slot_ids, n, num_slots);
}

int stepq_check_wait_timeout(int32_t *flag_out, stepq_stream stream)
{
    if (!flag_out) return STEPQ_INVALID_ARG;
    int *d_flag = nullptr;
    cudaError_t e = cudaMalloc(&d_flag, sizeof(int));
    if (e != cudaSuccess) return status_of(e);
    e = cudaMemsetAsync(d_flag, 0, sizeof(int), stream);
    if (e == cudaSuccess) e = stepq::launch_wait_check(d_flag, stream);
    int h = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&h, d_flag, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    const cudaError_t ef = cudaFree(d_flag);
    if (e == cudaSuccess) e = ef;
    if (e != cudaSuccess) return status_of(e);
    *flag_out = h;
    return STEPQ_OK;
}

int stepq_pool_get_error(stepq_pool *pool, int32_t *flag_out)
{
    if (!pool || !flag_out) return STEPQ_INVALID_ARG;
    int st = check_device(pool);
    if (st != STEPQ_OK) return st;
    int h = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(&h, pool->d_flag, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(pool->d_flag, 0, sizeof(int));
    if (e != cudaSuccess) return status_of(e);
    *flag_out = h;
    return STEPQ_OK;
}

}  // extern "C"
