// stepq_io.cu -- pool I/O kernels of libstepq (sm_100a): quantize fp32 states into the
// pool (clip-free dual-axis fit + round-half-even, STEPQuant summary "Method"), dequantize
// them back (FP16 pivot heads: round to binary16 and back), and copy packed slot images in
// and out.  One CTA of 256 threads per (request, head) state, each thread a 4-row x
// 16-column register tile.
#include <cfloat>
#include <cstdint>
#include <cuda_fp16.h>

#include "stepq_internal.h"
#include "stepq_tile.cuh"

namespace stepq {

constexpr int kIoRpStride = 12;     // padded row stride of the row-maxima exchange (floats)

// ------------------------------------------------------------------------------------------
// Fit + quantize + pack of a register tile (a state S).  On return S holds garbage.  Writes c (writer lanes), r (panel-0 threads)
// and the packed codes of the thread's rows.  Contains one __syncthreads (row maxima).
// `ok` is folded into that barrier: returns false on every thread if any thread passed false.
// ------------------------------------------------------------------------------------------
template <int ROWS, int BITS>
__device__ __forceinline__ bool fit_quantize_pack(float (&S)[ROWS][PANEL], const TileIdx<ROWS> &ix,
                                                  float *rp, float *xc, uint8_t *codes_out,
                                                  float *r_out, float *c_out, bool ok,
                                                  int n8 = 0, int n4 = 0, int pb = 0)
{
    // BITS == 0: per-key-row widths (stored rows 8-bit, 4-bit, 6-bit; panels of pb bytes)
    using L = Layout<ROWS>;

    // column maxima: max_i |S_ij| over the thread's rows, then over the LP lanes of the panel
    float cm[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; ++j) {
        float a = fabsf(S[0][j]);
#pragma unroll
        for (int m = 1; m < ROWS; m += 2)
            a = (m + 1 < ROWS) ? absmax3(a, S[m][j], S[m + 1][j]) : fmaxf(a, fabsf(S[m][j]));
        cm[j] = a;
    }
    reduce_scatter<PANEL, 4, L::LP / 2, true>(cm, ix.lane);
    float M = cm[0];
    int col;
    bool writer;
    if (L::LP == 32) {
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
        col = ix.lane >> 1;
        writer = (ix.lane & 1) == 0;
    } else {
        col = ix.rl;
        writer = true;
    }
    // c_j = sqrt(max_i |S_ij|) (correctly rounded); 1/c_j for the row fit (0 for a zero column)
    const float cnew = sqrtf(M);
    const float icn = cnew > 0.0f ? 1.0f / cnew : 0.0f;
    float *xcp = xc + ix.panel * PANEL;
    if (writer) {
        c_out[ix.panel * PANEL + col] = cnew;
        xcp[col] = icn;
    }
    __syncwarp();
    float ic[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(xcp + j);
        ic[j] = t.x; ic[j + 1] = t.y; ic[j + 2] = t.z; ic[j + 3] = t.w;
    }
    // P_ij = S_ij / c_j; per-thread row maxima of |P|
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            const float2 p = fmul2(make_float2(S[m][j], S[m][j + 1]), make_float2(ic[j], ic[j + 1]));
            S[m][j] = p.x;
            S[m][j + 1] = p.y;
        }
        float a = absmax3(S[m][0], S[m][1], S[m][2]);
#pragma unroll
        for (int j = 3; j < PANEL; j += 2)
            a = (j + 1 < PANEL) ? absmax3(a, S[m][j], S[m][j + 1]) : fmaxf(a, fabsf(S[m][j]));
        rp[ix.row(m) * kIoRpStride + ix.panel] = a;
    }
    if (__syncthreads_or(!ok)) return false;
    // r_i = max_j (|S_ij| / c_j) / qmax (correctly rounded division); quantize the rows
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        const int row = ix.row(m);
        const float4 a = *reinterpret_cast<const float4 *>(rp + row * kIoRpStride);
        const float4 b = *reinterpret_cast<const float4 *>(rp + row * kIoRpStride + 4);
        const float mr = max3(max3(a.x, a.y, a.z), max3(a.w, b.x, b.y), fmaxf(b.z, b.w));
        const int wdt = BITS ? BITS : row_width(row, n8, n4);
        const float MAG = kTwo23 + float(1 << (wdt - 1));
        const float r = mr / float(qmax_of(wdt));
        if (ix.panel == 0) r_out[row] = r;
        uint32_t u[PANEL];
        if (r >= FLT_MIN || r == 0.0f) {
            const float ir = r > 0.0f ? 1.0f / r : 0.0f;
            // fma(P, 1/r, 2^23 + 2^(b-1)) rounds P / r to the nearest integer, ties to even,
            // and leaves the offset-binary code in the low mantissa bits
#pragma unroll
            for (int j = 0; j < PANEL; j += 2) {
                const float2 f = ffma2(make_float2(S[m][j], S[m][j + 1]), make_float2(ir, ir),
                                       make_float2(MAG, MAG));
                u[j] = __float_as_uint(f.x);
                u[j + 1] = __float_as_uint(f.y);
            }
        } else {
            // subnormal row factor: 1/r would overflow; divide element by element
#pragma unroll
            for (int j = 0; j < PANEL; ++j) u[j] = __float_as_uint(S[m][j] / r + MAG);
        }
        if constexpr (BITS == 0) {
            uint8_t *seg = codes_out + ix.panel * pb + row_seg_off(row, n8, n4);
            if (wdt == 8)
                pack_seg<8>(u, seg);
            else if (wdt == 4)
                pack_seg<4>(u, seg);
            else
                pack_seg<6>(u, seg);
        } else {
            pack_seg<BITS>(u, codes_out + ix.panel * panel_bytes(BITS) + row * seg_bytes(BITS));
        }
    }
    return true;
}

// ------------------------------------------------------------------------------------------
// The impact-weighted fit (STEPQuant summary, "Method" para 4) of a register tile, in the
// order of its definition and with IEEE division and square root (w: the head's normalized
// row-impact weights):  r_i = sqrt(max_j |S_ij| / w_i);  c0_j = max_i |S_ij / r_i| / qmax;
// Q0 = nearest levels of S / (r c0);  c_j = sum_i w_i r_i Q0_ij S_ij / sum_i w_i r_i^2 Q0_ij^2
// (c0_j when a sum is not positive);  codes = nearest levels of S / (r c), clipped.
// ------------------------------------------------------------------------------------------
template <int BITS>
__device__ __forceinline__ void fit_quantize_pack_impact(float (&S)[4][PANEL], const TileIdx<4> &ix, float *rp,
                                                         const float *w, uint8_t *codes_out, float *r_out,
                                                         float *c_out)
{
    constexpr int QM = qmax_of(BITS);
    // row maxima of |S| over the panels
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float a = absmax3(S[m][0], S[m][1], S[m][2]);
#pragma unroll
        for (int j = 3; j < PANEL; j += 2)
            a = (j + 1 < PANEL) ? absmax3(a, S[m][j], S[m][j + 1]) : fmaxf(a, fabsf(S[m][j]));
        rp[ix.row(m) * kIoRpStride + ix.panel] = a;
    }
    __syncthreads();
    float r[4], P[4][PANEL];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int row = ix.row(m);
        const float4 a = *reinterpret_cast<const float4 *>(rp + row * kIoRpStride);
        const float4 b = *reinterpret_cast<const float4 *>(rp + row * kIoRpStride + 4);
        const float mr = max3(max3(a.x, a.y, a.z), max3(a.w, b.x, b.y), fmaxf(b.z, b.w));
        r[m] = sqrtf(mr / w[row]);
        if (ix.panel == 0) r_out[row] = r[m];
#pragma unroll
        for (int j = 0; j < PANEL; ++j) P[m][j] = r[m] > 0.0f ? S[m][j] / r[m] : 0.0f;
    }
    // per column (the warp holds all 128 rows of its panel): c0, the sums, c
    uint32_t u[4][PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; ++j) {
        const float mx = warp_absmax(fmaxf(absmax3(P[0][j], P[1][j], P[2][j]), fabsf(P[3][j])));
        const float c0 = mx / float(QM);
        float num = 0.0f, den = 0.0f;
        float q0[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            q0[m] = c0 > 0.0f ? fminf(fmaxf(rintf(P[m][j] / c0), -float(QM)), float(QM)) : 0.0f;
            const float wr = w[ix.row(m)] * r[m];
            num = fmaf(wr * q0[m], S[m][j], num);
            den = fmaf(wr * r[m] * q0[m], q0[m], den);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            num += __shfl_xor_sync(0xffffffffu, num, o);
            den += __shfl_xor_sync(0xffffffffu, den, o);
        }
        const float c = (num > 0.0f && den > 0.0f) ? num / den : c0;
        if (ix.lane == 0) c_out[ix.panel * PANEL + j] = c;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float q = c > 0.0f ? fminf(fmaxf(rintf(P[m][j] / c), -float(QM)), float(QM)) : 0.0f;
            u[m][j] = __float_as_uint(q + (kTwo23 + float(1 << (BITS - 1))));
        }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) pack_seg<BITS>(u[m], codes_out + ix.panel * panel_bytes(BITS) + ix.row(m) * seg_bytes(BITS));
}

// ------------------------------------------------------------------------------------------
// Pool I/O kernels: one CTA (256 threads, 4 x 16 tiles) per (request, head) state.
// ------------------------------------------------------------------------------------------
struct IoArgs {
    uint8_t *pool;
    long long slot_stride;
    const long long *head_off;
    const uint8_t *head_bits;
    int num_slots, H;
    const int32_t *slot_ids;
    int *flag;
    const float *impact;            // [H, d_k] normalized row-impact weights, or null (clip-free fit)
    const uint8_t *row_n8, *row_n4, *row_perm;  // heads with per-key-row widths (see the pool)
    const int32_t *row_pb;
};

template <int BITS>
__device__ __forceinline__ void load_fp32_item(const IoArgs &a, uint8_t *blk, const float *S,
                                               const TileIdx<4> &ix, float *rp, float *xc, int h)
{
    float T[4][PANEL];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int j = 0; j < PANEL; j += 4) {
            const float4 t = *reinterpret_cast<const float4 *>(S + ix.row(m) * DV + ix.panel * PANEL + j);
            T[m][j] = t.x; T[m][j + 1] = t.y; T[m][j + 2] = t.z; T[m][j + 3] = t.w;
        }
    float *r_out = reinterpret_cast<float *>(blk + codes_bytes(BITS));
    if (a.impact)
        fit_quantize_pack_impact<BITS>(T, ix, rp, a.impact + (long long)h * DK, blk, r_out, r_out + DK);
    else
        fit_quantize_pack<4, BITS>(T, ix, rp, xc, blk, r_out, r_out + DK, true);
}

__global__ void __launch_bounds__(256) load_fp32_kernel(const IoArgs a, const float *S)
{
    __shared__ __align__(16) float rp[DK * kIoRpStride];
    __shared__ __align__(16) float xc[NPANEL * PANEL];
    const long long it = blockIdx.x;
    const int b = int(it / a.H), h = int(it % a.H);
    const int slot = a.slot_ids[b];
    if (slot < 0 || slot >= a.num_slots) {
        if (threadIdx.x == 0) atomicOr(a.flag, STEPQ_FLAG_BAD_SLOT);
        return;
    }
    uint8_t *blk = a.pool + (long long)slot * a.slot_stride + a.head_off[h];
    const float *Si = S + it * DK * DV;
    const TileIdx<4> ix(threadIdx.x);
    switch (a.head_bits[h]) {
    case 0: {
        // per-key-row widths: stored row p holds key row perm[p]
        const int n8 = a.row_n8[h], n4 = a.row_n4[h], pb = a.row_pb[h];
        float T[4][PANEL];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int key = a.row_perm[h * DK + ix.row(m)];
#pragma unroll
            for (int j = 0; j < PANEL; j += 4) {
                const float4 t = *reinterpret_cast<const float4 *>(Si + key * DV + ix.panel * PANEL + j);
                T[m][j] = t.x; T[m][j + 1] = t.y; T[m][j + 2] = t.z; T[m][j + 3] = t.w;
            }
        }
        float *r_out = reinterpret_cast<float *>(blk + NPANEL * pb);
        fit_quantize_pack<4, 0>(T, ix, rp, xc, blk, r_out, r_out + DK, true, n8, n4, pb);
        break;
    }
    case 4: load_fp32_item<4>(a, blk, Si, ix, rp, xc, h); break;
    case 6: load_fp32_item<6>(a, blk, Si, ix, rp, xc, h); break;
    case 8: load_fp32_item<8>(a, blk, Si, ix, rp, xc, h); break;
    default: {
        // FP16 pivot head: the state rounded to binary16 (nearest, ties to even)
        __half *dst = reinterpret_cast<__half *>(blk);
        for (int e = threadIdx.x; e < DK * DV; e += blockDim.x) dst[e] = __float2half_rn(Si[e]);
    }
    }
}

template <int BITS>
__device__ __forceinline__ void dump_fp32_item(const uint8_t *blk, float *S, const TileIdx<4> &ix)
{
    const float *r = reinterpret_cast<const float *>(blk + codes_bytes(BITS));
    const float *c = r + DK;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int row = ix.row(m);
        float f[PANEL];
        load_codes<BITS>(blk + ix.panel * panel_bytes(BITS) + row * seg_bytes(BITS), f);
        const double rr = r[row];
#pragma unroll
        for (int j = 0; j < PANEL; j += 4) {
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int jj = j + e;
                // Q * r * c is exact in double; one rounding to float
                const double code = double(f[jj]) / double(pos_scale(BITS, jj));
                o[e] = float(code * rr * double(c[ix.panel * PANEL + jj]));
            }
            *reinterpret_cast<float4 *>(S + row * DV + ix.panel * PANEL + j) = make_float4(o[0], o[1], o[2], o[3]);
        }
    }
}

__global__ void __launch_bounds__(256) dump_fp32_kernel(const IoArgs a, float *S)
{
    const long long it = blockIdx.x;
    const int b = int(it / a.H), h = int(it % a.H);
    const int slot = a.slot_ids[b];
    if (slot < 0 || slot >= a.num_slots) {
        if (threadIdx.x == 0) atomicOr(a.flag, STEPQ_FLAG_BAD_SLOT);
        return;
    }
    const uint8_t *blk = a.pool + (long long)slot * a.slot_stride + a.head_off[h];
    float *Si = S + it * DK * DV;
    const TileIdx<4> ix(threadIdx.x);
    switch (a.head_bits[h]) {
    case 0: {
        const int n8 = a.row_n8[h], n4 = a.row_n4[h], pb = a.row_pb[h];
        const float *r = reinterpret_cast<const float *>(blk + NPANEL * pb);
        const float *c = r + DK;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int p = ix.row(m);
            const int key = a.row_perm[h * DK + p];
            const int wdt = row_width(p, n8, n4);
            const uint8_t *seg = blk + ix.panel * pb + row_seg_off(p, n8, n4);
            float f[PANEL];
            if (wdt == 8)
                load_codes_unscaled<8>(seg, f);
            else if (wdt == 4)
                load_codes_unscaled<4>(seg, f);
            else
                load_codes_unscaled<6>(seg, f);
            const double rr = r[p];
#pragma unroll
            for (int j = 0; j < PANEL; ++j)       // (Q r) c in double, Q r exact
                Si[key * DV + ix.panel * PANEL + j] = float(double(f[j]) * rr * double(c[ix.panel * PANEL + j]));
        }
        break;
    }
    case 4: dump_fp32_item<4>(blk, Si, ix); break;
    case 6: dump_fp32_item<6>(blk, Si, ix); break;
    case 8: dump_fp32_item<8>(blk, Si, ix); break;
    default: {
        const __half *src = reinterpret_cast<const __half *>(blk);
        for (int e = threadIdx.x; e < DK * DV; e += blockDim.x) Si[e] = __half2float(src[e]);
    }
    }
}

// Copy whole slot images between the pool and a dense [n, slot_stride] buffer.
__global__ void copy_slots_kernel(const IoArgs a, const uint8_t *src, uint8_t *dst, int into_pool)
{
    const int b = blockIdx.y;
    const int slot = a.slot_ids[b];
    if (slot < 0 || slot >= a.num_slots) {
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.flag, STEPQ_FLAG_BAD_SLOT);
        return;
    }
    const long long words = a.slot_stride / 16;
    const uint4 *s = reinterpret_cast<const uint4 *>(into_pool ? src + (long long)b * a.slot_stride
                                                               : a.pool + (long long)slot * a.slot_stride);
    uint4 *d = reinterpret_cast<uint4 *>(into_pool ? a.pool + (long long)slot * a.slot_stride
                                                   : dst + (long long)b * a.slot_stride);
    for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < words;
         w += (long long)gridDim.x * blockDim.x)
        d[w] = s[w];
}

// ------------------------------------------------------------------------------------------
// The bounded-wait path of the kernels, on its own: one warp waits on a shared-memory
// mbarrier that nothing completes (no copy is in flight), gives up after a short poll limit,
// raises the timeout bit of the flag and returns -- the same steps a decode CTA takes when a
// stage never arrives, with a limit short enough for a health check.
// ------------------------------------------------------------------------------------------
__global__ void wait_check_kernel(int *flag)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncwarp();
    const bool ok = mbar_wait_bounded<1024>(&bar, 0u);
    if (threadIdx.x == 0) {
        if (!ok) atomicOr(flag, STEPQ_FLAG_TIMEOUT);
        mbar_arrive(&bar);                         // leave the barrier in a completed phase
    }
}

// ------------------------------------------------------------------------------------------
// Launchers
// ------------------------------------------------------------------------------------------
namespace {

IoArgs io_args(const stepq_pool *p, const int32_t *slot_ids)
{
    IoArgs a;
    a.pool = p->d_pool;
    a.slot_stride = p->slot_stride;
    a.head_off = p->d_offs;
    a.head_bits = p->d_bits;
    a.num_slots = p->num_slots;
    a.H = p->H;
    a.slot_ids = slot_ids;
    a.flag = p->d_flag;
    a.impact = p->d_impact;
    a.row_n8 = p->d_rn8;
    a.row_n4 = p->d_rn4;
    a.row_perm = p->d_perm;
    a.row_pb = p->d_rpb;
    return a;
}

}  // namespace

cudaError_t launch_wait_check(int *flag, cudaStream_t stream)
{
    wait_check_kernel<<<1, 32, 0, stream>>>(flag);
    return cudaGetLastError();
}

cudaError_t launch_load_fp32(const stepq_pool *p, const int32_t *slot_ids, int n, const float *S,
                             cudaStream_t stream)
{
    load_fp32_kernel<<<dim3(unsigned(n) * p->H), 256, 0, stream>>>(io_args(p, slot_ids), S);
    return cudaGetLastError();
}

cudaError_t launch_dump_fp32(const stepq_pool *p, const int32_t *slot_ids, int n, float *S, cudaStream_t stream)
{
    dump_fp32_kernel<<<dim3(unsigned(n) * p->H), 256, 0, stream>>>(io_args(p, slot_ids), S);
    return cudaGetLastError();
}

cudaError_t launch_copy_slots(const stepq_pool *p, const int32_t *slot_ids, int n, const uint8_t *src,
                              uint8_t *dst, bool into_pool, cudaStream_t stream)
{
    const long long words = p->slot_stride / 16;
    const int bx = int((words + 255) / 256 < 64 ? (words + 255) / 256 : 64);
    copy_slots_kernel<<<dim3(bx, n), 256, 0, stream>>>(io_args(p, slot_ids), src, dst, into_pool ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace stepq
