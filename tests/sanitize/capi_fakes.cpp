// capi_fakes.cpp -- host-side checks of the C ABI under AddressSanitizer, LeakSanitizer and
// UndefinedBehaviorSanitizer, with no GPU.
//
// The library's host code (stepq_capi.cu, stepq_alloc.cpp) is linked against the fakes below
// instead of the CUDA runtime: "device" memory is host memory from malloc, copies are memcpy,
// streams and events are small heap objects, and the kernel launchers record their calls.
// Failures are made on the host by the fakes themselves (an allocation that fails on
// request), so the error paths of the library run for real and every buffer they leak
// shows up in LeakSanitizer's report at exit.
//
// Built and run by tests/test_sanitizers.py; exit status 0 means every check passed.
#include <cuda_runtime_api.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <random>
#include <set>
#include <vector>

#include "stepq.h"
#include "stepq_internal.h"

// ------------------------------------------------------------------ fake CUDA runtime

namespace fake {
int malloc_calls = 0;          // successful and failed cudaMalloc calls
int fail_malloc_at = -1;       // index of the cudaMalloc call that fails (-1: none)
int handle_calls = 0;          // stream and event creations
int fail_handle_at = -1;
std::set<void *> live;         // fake device allocations not yet freed
std::set<void *> handles;      // live streams and events
int launches = 0;
int h2d_copies = 0;            // cudaMemcpyAsync calls from host to device
const int32_t *last_slots = nullptr;
int last_n = 0;
const void *last_q = nullptr;
}  // namespace fake

extern "C" {

cudaError_t cudaMalloc(void **p, size_t n)
{
    const int k = fake::malloc_calls++;
    if (k == fake::fail_malloc_at) {
        *p = nullptr;
        return cudaErrorMemoryAllocation;
    }
    *p = std::malloc(n ? n : 1);
    if (!*p) return cudaErrorMemoryAllocation;
    fake::live.insert(*p);
    return cudaSuccess;
}

cudaError_t cudaFree(void *p)
{
    if (!p) return cudaSuccess;
    if (!fake::live.erase(p)) return cudaErrorInvalidValue;        // double or foreign free
    std::free(p);
    return cudaSuccess;
}

cudaError_t cudaGetDevice(int *d)
{
    *d = 0;
    return cudaSuccess;
}

cudaError_t cudaDeviceGetAttribute(int *v, cudaDeviceAttr, int)
{
    *v = 148;
    return cudaSuccess;
}

static cudaError_t new_handle(void **h)
{
    const int k = fake::handle_calls++;
    if (k == fake::fail_handle_at) return cudaErrorMemoryAllocation;
    *h = std::malloc(16);
    fake::handles.insert(*h);
    return cudaSuccess;
}

static cudaError_t free_handle(void *h)
{
    if (!fake::handles.erase(h)) return cudaErrorInvalidResourceHandle;
    std::free(h);
    return cudaSuccess;
}

cudaError_t cudaStreamCreateWithFlags(cudaStream_t *s, unsigned int)
{
    return new_handle(reinterpret_cast<void **>(s));
}
cudaError_t cudaStreamDestroy(cudaStream_t s) { return free_handle(s); }
cudaError_t cudaEventCreateWithFlags(cudaEvent_t *e, unsigned int)
{
    return new_handle(reinterpret_cast<void **>(e));
}
cudaError_t cudaEventDestroy(cudaEvent_t e) { return free_handle(e); }
cudaError_t cudaEventRecord(cudaEvent_t, cudaStream_t) { return cudaSuccess; }
cudaError_t cudaEventSynchronize(cudaEvent_t) { return cudaSuccess; }
cudaError_t cudaStreamWaitEvent(cudaStream_t, cudaEvent_t, unsigned int) { return cudaSuccess; }
cudaError_t cudaStreamSynchronize(cudaStream_t) { return cudaSuccess; }
cudaError_t cudaDeviceSynchronize(void) { return cudaSuccess; }

cudaError_t cudaMemset(void *p, int v, size_t n)
{
    std::memset(p, v, n);
    return cudaSuccess;
}
cudaError_t cudaMemsetAsync(void *p, int v, size_t n, cudaStream_t)
{
    std::memset(p, v, n);
    return cudaSuccess;
}
cudaError_t cudaMemcpy(void *d, const void *s, size_t n, cudaMemcpyKind)
{
    std::memcpy(d, s, n);
    return cudaSuccess;
}
cudaError_t cudaMemcpyAsync(void *d, const void *s, size_t n, cudaMemcpyKind kind, cudaStream_t)
{
    if (kind == cudaMemcpyHostToDevice) ++fake::h2d_copies;
    std::memcpy(d, s, n);
    return cudaSuccess;
}

// fat-binary registration of the compiled translation unit (it holds no kernels)
void **__cudaRegisterFatBinary(void *) { static void *h = nullptr; return &h; }
void __cudaRegisterFatBinaryEnd(void **) {}
void __cudaUnregisterFatBinary(void **) {}

}  // extern "C"

// ------------------------------------------------------------------ fake kernel launchers

namespace stepq {
cudaError_t decode_configure(stepq_pool *p)
{
    p->decode_grid = 2 * p->num_sms;
    p->decode_smem = 1;
    return cudaSuccess;
}
cudaError_t launch_decode(const stepq_pool *, const int32_t *slot_ids, int n, const void *q, const void *,
                          const void *, const void *, const void *, float *, cudaStream_t)
{
    ++fake::launches;
    fake::last_slots = slot_ids;
    fake::last_n = n;
    fake::last_q = q;
    return cudaSuccess;
}
cudaError_t launch_wait_check(int *flag, cudaStream_t)
{
    *flag = STEPQ_FLAG_TIMEOUT;
    return cudaSuccess;
}
cudaError_t launch_load_fp32(const stepq_pool *, const int32_t *, int, const float *, cudaStream_t)
{
    ++fake::launches;
    return cudaSuccess;
}
cudaError_t launch_dump_fp32(const stepq_pool *, const int32_t *, int, float *, cudaStream_t)
{
    ++fake::launches;
    return cudaSuccess;
}
cudaError_t launch_copy_slots(const stepq_pool *, const int32_t *, int, const uint8_t *, uint8_t *, bool,
                              cudaStream_t)
{
    ++fake::launches;
    return cudaSuccess;
}
}  // namespace stepq

// ------------------------------------------------------------------ checks

static int failures = 0, checks = 0;
#define CHECK(cond)                                                                   \
    do {                                                                              \
        ++checks;                                                                     \
        if (!(cond)) {                                                                \
            ++failures;                                                               \
            std::fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
        }                                                                             \
    } while (0)

static stepq_pool_desc desc_of(std::vector<uint8_t> &bits, int slots, int hk, int gate, int dtype)
{
    stepq_pool_desc d;
    d.num_slots = slots;
    d.num_heads = int32_t(bits.size());
    d.num_key_heads = hk;
    d.d_k = 128;
    d.d_v = 128;
    d.gate_mode = gate;
    d.in_dtype = dtype;
    d.head_bits = bits.data();
    return d;
}

static size_t block_of(int b) { return b == 16 ? 32768 : size_t(128 * 128 * b / 8 + 1024); }

// Every kind of pool is created and destroyed; sizes and offsets follow the documented layout.
static void test_create_destroy()
{
    std::vector<std::vector<uint8_t>> cfgs = {{4, 6, 8, 8}, {6, 16, 4, 8}, {8}, {4, 4, 4, 4, 6, 6, 8, 16}};
    for (auto &bits : cfgs) {
        for (int gate = 0; gate < 2; ++gate) {
            stepq_pool_desc d = desc_of(bits, 3, 1, gate, gate);
            stepq_pool *p = nullptr;
            CHECK(stepq_pool_create(&d, &p) == STEPQ_OK && p);
            size_t stride = 0, total = 0, expect = 0;
            CHECK(stepq_pool_bytes(p, &stride, &total) == STEPQ_OK);
            for (size_t h = 0; h < bits.size(); ++h) {
                size_t off = 0;
                CHECK(stepq_pool_head_offset(p, int32_t(h), &off) == STEPQ_OK && off == expect);
                expect += block_of(bits[h]);
            }
            CHECK(stride == expect && total == 3 * expect);
            size_t off = 0;
            CHECK(stepq_pool_head_offset(p, int32_t(bits.size()), &off) == STEPQ_INVALID_ARG);
            CHECK(stepq_pool_destroy(p) == STEPQ_OK);
        }
    }
    CHECK(fake::live.empty() && fake::handles.empty());
}

// Per-key-row pools: block bytes 8 * roundup16(16 n8 + 8 n4 + 12 n6) + 1024.
static void test_rows_pool()
{
    std::vector<uint8_t> bits = {0, 6, 0};
    std::vector<uint8_t> rb(3 * 128, 6);
    for (int i = 0; i < 128; ++i) rb[i] = uint8_t(i % 3 == 0 ? 8 : i % 3 == 1 ? 4 : 6);
    for (int i = 0; i < 128; ++i) rb[256 + i] = 4;
    stepq_pool_desc d = desc_of(bits, 2, 3, 1, 1);
    stepq_pool *p = nullptr;
    CHECK(stepq_pool_create_rows(&d, rb.data(), &p) == STEPQ_OK);
    int n8 = 0, n4 = 0, n6 = 0;
    for (int i = 0; i < 128; ++i) (rb[i] == 8 ? n8 : rb[i] == 4 ? n4 : n6) += 1;
    const size_t b0 = size_t(8 * ((16 * n8 + 8 * n4 + 12 * n6 + 15) / 16 * 16) + 1024);
    const size_t b2 = size_t(8 * (8 * 128) + 1024);
    size_t stride = 0;
    CHECK(stepq_pool_bytes(p, &stride, nullptr) == STEPQ_OK && stride == b0 + block_of(6) + b2);
    CHECK(stepq_pool_destroy(p) == STEPQ_OK);
    rb[5] = 5;                                                       // not a row width
    CHECK(stepq_pool_create_rows(&d, rb.data(), &p) == STEPQ_UNSUPPORTED && !p);
    CHECK(stepq_pool_create_rows(&d, nullptr, &p) == STEPQ_INVALID_ARG);
    CHECK(fake::live.empty() && fake::handles.empty());
}

// Each device allocation of pool creation fails in turn: STEPQ_OUT_OF_MEMORY, no pool, and
// every allocation made before the failure is released.  The same for the pivot stream and
// events (their failure is a CUDA error).
static void test_injected_allocation_failures()
{
    for (int rows = 0; rows < 2; ++rows) {
        std::vector<uint8_t> bits = rows ? std::vector<uint8_t>{0, 16, 8} : std::vector<uint8_t>{4, 16, 8};
        std::vector<uint8_t> rb(bits.size() * 128, 4);
        stepq_pool_desc d = desc_of(bits, 4, 1, 1, 1);
        auto create = [&](stepq_pool **p) {
            return rows ? stepq_pool_create_rows(&d, rb.data(), p) : stepq_pool_create(&d, p);
        };
        fake::malloc_calls = 0;
        stepq_pool *p = nullptr;
        CHECK(create(&p) == STEPQ_OK);
        const int n_alloc = fake::malloc_calls;
        CHECK(n_alloc >= 5);
        CHECK(stepq_pool_destroy(p) == STEPQ_OK);
        for (int k = 0; k < n_alloc; ++k) {
            fake::malloc_calls = 0;
            fake::fail_malloc_at = k;
            p = reinterpret_cast<stepq_pool *>(&d);                  // must be overwritten
            CHECK(create(&p) == STEPQ_OUT_OF_MEMORY);
            CHECK(p == nullptr);
            CHECK(fake::live.empty() && fake::handles.empty());
        }
        fake::fail_malloc_at = -1;
        for (int k = 0; k < 3; ++k) {                                // pivot stream, fork and join events
            fake::handle_calls = 0;
            fake::fail_handle_at = k;
            p = nullptr;
            CHECK(create(&p) == STEPQ_OUT_OF_MEMORY && p == nullptr);
            CHECK(fake::live.empty() && fake::handles.empty());
        }
        fake::fail_handle_at = -1;
    }
}

static void test_impact_scores()
{
    std::vector<uint8_t> bits = {4, 6};
    stepq_pool_desc d = desc_of(bits, 2, 2, 0, 1);
    stepq_pool *p = nullptr;
    CHECK(stepq_pool_create(&d, &p) == STEPQ_OK);
    std::vector<float> om(2 * 128);
    std::mt19937 g(5);
    std::lognormal_distribution<float> ln(0.0f, 1.2f);
    for (auto &x : om) x = ln(g);
    CHECK(stepq_pool_set_impact(p, om.data()) == STEPQ_OK && p->d_impact);
    for (int h = 0; h < 2; ++h) {                                     // w = omega / mean(omega), in double
        double sum = 0.0;
        for (int i = 0; i < 128; ++i) sum += om[h * 128 + i];
        for (int i = 0; i < 128; ++i)
            CHECK(p->d_impact[h * 128 + i] == float(double(om[h * 128 + i]) / (sum / 128.0)));
    }
    const float bad[3] = {0.0f, -1.0f, INFINITY};
    for (float b : bad) {
        std::vector<float> o2 = om;
        o2[77] = b;
        CHECK(stepq_pool_set_impact(p, o2.data()) == STEPQ_INVALID_ARG);
    }
    std::vector<float> o3 = om;
    o3[3] = NAN;
    CHECK(stepq_pool_set_impact(p, o3.data()) == STEPQ_INVALID_ARG);
    CHECK(stepq_pool_set_impact(p, nullptr) == STEPQ_OK && !p->d_impact);
    CHECK(stepq_pool_destroy(p) == STEPQ_OK);
    CHECK(fake::live.empty());
}

// The debug mode rejects duplicate and out-of-range slot ids before any launch; without it
// the ids go to the kernels unchecked.
static void test_debug_slots()
{
    std::vector<uint8_t> bits = {4, 8};
    stepq_pool_desc d = desc_of(bits, 8, 1, 0, 1);
    stepq_pool *p = nullptr;
    CHECK(stepq_pool_create(&d, &p) == STEPQ_OK);
    alignas(16) static uint16_t q[4 * 128], k[4 * 128], v[4 * 2 * 128], a[4 * 2], be[4 * 2];
    alignas(16) static float y[4 * 2 * 128], S[4 * 2 * 128 * 128];
    alignas(16) static uint8_t img[4 * 30000];
    int32_t *ids = nullptr;
    CHECK(cudaMalloc(reinterpret_cast<void **>(&ids), 16) == cudaSuccess);
    const int32_t dup[3] = {3, 1, 3}, good[3] = {3, 1, 2}, out[2] = {0, 8};
    auto step = [&](const int32_t *host, int n) {
        std::memcpy(ids, host, sizeof(int32_t) * n);
        return stepq_decode_step(p, ids, n, q, k, v, a, be, y, nullptr);
    };
    CHECK(stepq_pool_set_debug(p, 2) == STEPQ_INVALID_ARG);
    CHECK(stepq_pool_set_debug(p, STEPQ_DEBUG_SLOTS) == STEPQ_OK);
    int before = fake::launches;
    CHECK(step(dup, 3) == STEPQ_INVALID_ARG);
    CHECK(step(out, 2) == STEPQ_INVALID_ARG);
    std::memcpy(ids, dup, sizeof(dup));
    CHECK(stepq_pool_load_fp32(p, ids, 3, S, nullptr) == STEPQ_INVALID_ARG);
    CHECK(stepq_pool_dump_fp32(p, ids, 3, S, nullptr) == STEPQ_INVALID_ARG);
    CHECK(stepq_pool_load_packed(p, ids, 3, img, nullptr) == STEPQ_INVALID_ARG);
    CHECK(stepq_pool_dump_packed(p, ids, 3, img, nullptr) == STEPQ_INVALID_ARG);
    CHECK(stepq_decode_step_host(p, dup, 3, q, k, v, a, be, y, nullptr) == STEPQ_INVALID_ARG);
    CHECK(fake::launches == before);
    CHECK(step(good, 3) == STEPQ_OK && fake::launches == before + 1);
    CHECK(stepq_decode_step_host(p, good, 3, q, k, v, a, be, y, nullptr) == STEPQ_OK);
    CHECK(stepq_pool_set_debug(p, 0) == STEPQ_OK);
    CHECK(step(dup, 3) == STEPQ_OK);                                 // unchecked: left to the caller
    CHECK(cudaFree(ids) == cudaSuccess);
    CHECK(stepq_pool_destroy(p) == STEPQ_OK);
    CHECK(fake::live.empty() && fake::handles.empty());

    CHECK(stepq_check_slot_ids(good, 3, 4) == STEPQ_OK);
    CHECK(stepq_check_slot_ids(good, 3, 3) == STEPQ_INVALID_ARG);
    CHECK(stepq_check_slot_ids(dup, 3, 8) == STEPQ_INVALID_ARG);
    CHECK(stepq_check_slot_ids(nullptr, 0, 8) == STEPQ_OK);
    CHECK(stepq_check_slot_ids(nullptr, 2, 8) == STEPQ_INVALID_ARG);
    CHECK(stepq_check_slot_ids(good, -1, 8) == STEPQ_INVALID_ARG);
    CHECK(stepq_check_slot_ids(good, 3, 0) == STEPQ_INVALID_ARG);
}

// The host-buffer path copies each call's inputs into a staging buffer of the pool and hands
// the kernel pointers into it; consecutive calls alternate between two buffers, which grow
// when a call has more requests than any before.
static void test_host_path_staging()
{
    std::vector<uint8_t> bits = {6, 6, 8, 4};
    stepq_pool_desc d = desc_of(bits, 64, 2, 1, 1);                  // KDA, bf16: alpha [n, H, 128]
    stepq_pool *p = nullptr;
    CHECK(stepq_pool_create(&d, &p) == STEPQ_OK);
    for (int call = 0; call < 5; ++call) {
        const int n = call < 2 ? 3 : 17 + call;
        std::vector<int32_t> ids(n);
        for (int i = 0; i < n; ++i) ids[i] = (7 * i + call) % 64;
        std::vector<uint16_t> q(size_t(n) * 2 * 128), k(q.size()), v(size_t(n) * 4 * 128), a(v.size()), b(size_t(n) * 4);
        for (size_t i = 0; i < q.size(); ++i) q[i] = uint16_t(i * 3 + call);
        std::vector<float> y(size_t(n) * 4 * 128, -1.0f);
        CHECK(stepq_decode_step_host(p, ids.data(), n, q.data(), k.data(), v.data(), a.data(), b.data(), y.data(),
                                     nullptr) == STEPQ_OK);
        CHECK(fake::last_n == n && std::memcmp(fake::last_slots, ids.data(), sizeof(int32_t) * n) == 0);
        CHECK(std::memcmp(fake::last_q, q.data(), q.size() * 2) == 0);
        const uint8_t *stage = p->d_host_stage[call & 1];
        CHECK(reinterpret_cast<const uint8_t *>(fake::last_q) > stage &&
              reinterpret_cast<const uint8_t *>(fake::last_q) < stage + p->host_stage_cap);
    }
    // inputs placed at the offsets of stepq_host_image_layout: one host-to-device copy, same data
    for (int n : {1, 9, 64}) {
        size_t off[6] = {0}, total = 0;
        CHECK(stepq_host_image_layout(p, n, off, &total) == STEPQ_OK);
        CHECK(off[0] == 0 && total > off[5]);
        for (int i = 1; i < 6; ++i) CHECK(off[i] % 256 == 0 && off[i] > off[i - 1]);
        std::vector<uint8_t> image(total, 0);
        int32_t *ids = reinterpret_cast<int32_t *>(image.data());
        for (int i = 0; i < n; ++i) ids[i] = (5 * i + 3) % 64;
        for (size_t e = off[1]; e < total; ++e) image[e] = uint8_t(e * 7 + n);
        std::vector<float> y(size_t(n) * 4 * 128);
        const uint8_t *I = image.data();
        const int before = fake::h2d_copies;
        CHECK(stepq_decode_step_host(p, ids, n, I + off[1], I + off[2], I + off[3], I + off[4], I + off[5],
                                     y.data(), nullptr) == STEPQ_OK);
        CHECK(fake::h2d_copies == before + 1);
        CHECK(std::memcmp(fake::last_slots, ids, sizeof(int32_t) * n) == 0);
        CHECK(std::memcmp(fake::last_q, I + off[1], off[2] - off[1]) == 0);
        // one array elsewhere: six copies
        std::vector<uint8_t> other(I + off[3], I + off[4]);
        const int before6 = fake::h2d_copies;
        CHECK(stepq_decode_step_host(p, ids, n, I + off[1], I + off[2], other.data(), I + off[4], I + off[5],
                                     y.data(), nullptr) == STEPQ_OK);
        CHECK(fake::h2d_copies == before6 + 6);
    }
    size_t off[6];
    CHECK(stepq_host_image_layout(p, 65, off, nullptr) == STEPQ_INVALID_ARG);
    CHECK(stepq_host_image_layout(p, 2, nullptr, nullptr) == STEPQ_INVALID_ARG);
    CHECK(stepq_pool_host_wait(p, nullptr) == STEPQ_OK);
    CHECK(stepq_pool_destroy(p) == STEPQ_OK);
    CHECK(fake::live.empty() && fake::handles.empty());
}

static void test_argument_checks()
{
    std::vector<uint8_t> bits = {4, 6, 8, 5};
    stepq_pool_desc d = desc_of(bits, 4, 2, 0, 1);
    stepq_pool *p = nullptr;
    CHECK(stepq_pool_create(nullptr, &p) == STEPQ_INVALID_ARG);
    CHECK(stepq_pool_create(&d, &p) == STEPQ_UNSUPPORTED);           // width 5
    bits[3] = 8;
    d.num_key_heads = 3;
    CHECK(stepq_pool_create(&d, &p) == STEPQ_INVALID_ARG);           // H_k does not divide H
    d.num_key_heads = 2;
    d.d_v = 64;
    CHECK(stepq_pool_create(&d, &p) == STEPQ_UNSUPPORTED);
    d.d_v = 128;
    std::vector<uint8_t> many(257, 4);
    stepq_pool_desc dm = desc_of(many, 4, 1, 0, 1);
    CHECK(stepq_pool_create(&dm, &p) == STEPQ_UNSUPPORTED);
    CHECK(stepq_pool_create(&d, &p) == STEPQ_OK);
    alignas(16) static uint8_t buf[64];
    int32_t *ids = nullptr;
    CHECK(cudaMalloc(reinterpret_cast<void **>(&ids), 16) == cudaSuccess);
    CHECK(stepq_decode_step(p, ids, 5, buf, buf, buf, buf, buf, reinterpret_cast<float *>(buf), nullptr) ==
          STEPQ_INVALID_ARG);                                        // n > num_slots
    CHECK(stepq_decode_step(p, ids, 2, buf + 4, buf, buf, buf, buf, reinterpret_cast<float *>(buf), nullptr) ==
          STEPQ_INVALID_ARG);                                        // q not 16-byte aligned
    CHECK(stepq_decode_step(p, ids, 0, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr) == STEPQ_OK);
    int32_t flag = -1;
    CHECK(stepq_check_wait_timeout(&flag, nullptr) == STEPQ_OK && flag == STEPQ_FLAG_TIMEOUT);
    CHECK(stepq_pool_get_error(p, &flag) == STEPQ_OK && flag == 0);
    CHECK(cudaFree(ids) == cudaSuccess);
    CHECK(stepq_pool_destroy(p) == STEPQ_OK);
    CHECK(stepq_pool_destroy(nullptr) == STEPQ_OK);
    for (int st = -6; st <= 1; ++st) CHECK(stepq_status_string(st) != nullptr);
    CHECK(fake::live.empty() && fake::handles.empty());
}

// The allocator on random inputs: widths from the candidates, budget kept, pivots counted;
// and its argument errors.
static void test_allocator()
{
    std::mt19937_64 g(11);
    std::uniform_real_distribution<double> u(0.0, std::log(4096.0));
    const uint8_t cand[3] = {4, 6, 8};
    for (int trial = 0; trial < 200; ++trial) {
        const int N = 1 + int(g() % 300);
        std::vector<double> hl(N), dist(size_t(N) * 3);
        for (auto &h : hl) h = std::exp(u(g));
        for (auto &x : dist) x = std::exp(u(g) - 6.0);
        const double avg = 4.0 + double(g() % 41) / 10.0;
        const int npiv = int(g() % 4) % (N + 1);
        std::vector<uint8_t> out(N, 0);
        const bool use_d = trial & 1;
        int st = stepq_allocate_bits_pivots(hl.data(), use_d ? dist.data() : nullptr, N, cand, 3, avg, npiv, out.data());
        CHECK(st == STEPQ_OK);
        long sum = 0;
        int piv = 0;
        for (int i = 0; i < N; ++i) {
            CHECK(out[i] == 4 || out[i] == 6 || out[i] == 8 || out[i] == 16);
            if (out[i] == 16) ++piv; else sum += out[i];
        }
        CHECK(piv == npiv && sum <= long(std::floor((N - npiv) * avg + 1e-9)));
    }
    std::vector<double> hl = {1.0, 2.0, 3.0};
    std::vector<uint8_t> out(3);
    CHECK(stepq_allocate_bits(hl.data(), nullptr, 3, cand, 3, 3.0, out.data()) == STEPQ_INVALID_ARG);
    hl[1] = -1.0;
    CHECK(stepq_allocate_bits(hl.data(), nullptr, 3, cand, 3, 6.0, out.data()) == STEPQ_INVALID_ARG);
    hl[1] = NAN;
    CHECK(stepq_allocate_bits(hl.data(), nullptr, 3, cand, 3, 6.0, out.data()) == STEPQ_INVALID_ARG);
    CHECK(stepq_allocate_bits(nullptr, nullptr, 3, cand, 3, 6.0, out.data()) == STEPQ_INVALID_ARG);
    CHECK(stepq_allocate_bits(hl.data(), nullptr, 0, cand, 3, 6.0, out.data()) == STEPQ_INVALID_ARG);
}

int main()
{
    test_argument_checks();
    test_create_destroy();
    test_rows_pool();
    test_injected_allocation_failures();
    test_impact_scores();
    test_debug_slots();
    test_host_path_staging();
    test_allocator();
    std::printf("%d checks, %d failures\n", checks, failures);
    return failures ? 1 : 0;
}
