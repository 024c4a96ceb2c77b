// stepq_tile.cuh -- the per-thread register tile of one 128 x 128 state and the
// arithmetic on it: unpacking codes, the clip-free dual-axis fit, round-half-even
// quantization and repacking.  Shared by the decode, load and dump kernels.
//
// Tile: a state is split into 8 panels of 16 columns (the packed stream is
// panel-major).  A thread owns ROWS rows x one panel (16 columns), i.e. ROWS*16
// elements held in registers; LP = 128 / ROWS lanes share a panel, PW = 32 / LP
// panels share a warp.  ROWS = 4: 256 threads / state; ROWS = 8: 128 threads.
#pragma once

#include <cstdint>
#include "stepq_device.cuh"

namespace stepq {

constexpr int DK = 128;
constexpr int DV = 128;
constexpr int PANEL = 16;
constexpr int NPANEL = DV / PANEL;

__host__ __device__ constexpr int qmax_of(int bits) { return (1 << (bits - 1)) - 1; }
__host__ __device__ constexpr int codes_bytes(int bits) { return DK * DV * bits / 8; }
// head block: codes + r + c; an FP16 pivot head (width 16) holds the state as binary16 values
__host__ __device__ constexpr int block_bytes(int bits)
{
    return bits == 16 ? 2 * DK * DV : codes_bytes(bits) + 4 * DK + 4 * DV;
}
// bytes of one row's 16 codes inside a panel, and the panel size
__host__ __device__ constexpr int seg_bytes(int bits) { return PANEL * bits / 8; }
__host__ __device__ constexpr int panel_bytes(int bits) { return DK * seg_bytes(bits); }

// Unpacked codes come out multiplied by a power of two that depends on the column's
// position in the panel (the field is read in place from the packed word).  The
// tile folds 1/scale into the column scale, so the products stay exact.
__host__ __device__ constexpr float pos_scale(int bits, int p)
{
    return bits == 8 ? 1.0f
         : bits == 6 ? ((p & 3) == 0 ? 1.0f : (p & 3) == 2 ? 4096.0f : 64.0f)
                     : ((p & 7) == 0 ? 1.0f : (p & 7) == 1 ? 16.0f : (p & 7) == 2 ? 256.0f
                        : (p & 7) == 3 ? 4096.0f : (p & 7) == 4 ? 65536.0f : (p & 7) == 5 ? 16.0f
                        : (p & 7) == 6 ? 256.0f : 4096.0f);
}

constexpr uint32_t kMagicBits = 0x4B000000u;     // bit pattern of 2^23
constexpr float kTwo23 = 8388608.0f;

// Bias that turns the float 2^23 + u * s (u the offset-binary field) into code * s.
__host__ __device__ constexpr float pos_bias(int bits, int p)
{
    return kTwo23 + float(1 << (bits - 1)) * pos_scale(bits, p);
}

// ---------------------------------------------------------------- unpack one row segment

// (a & mask) | magic in one three-input logic op; both constants are register operands
// (a logic op encodes at most one immediate).
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t mask, uint32_t magic)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
    return d;
}

template <int BITS>
__device__ __forceinline__ void unpack_seg(const uint8_t *seg, float (&f)[PANEL]);

template <>
__device__ __forceinline__ void unpack_seg<8>(const uint8_t *seg, float (&f)[PANEL])
{
    const uint4 w = *reinterpret_cast<const uint4 *>(seg);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            f[4 * t + e] = __uint_as_float(__byte_perm(ws[t], kMagicBits, 0x7540u | e));
}

template <>
__device__ __forceinline__ void unpack_seg<4>(const uint8_t *seg, float (&f)[PANEL])
{
    const uint2 w = *reinterpret_cast<const uint2 *>(seg);
    const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const uint32_t lo = ws[t], hi = ws[t] >> 16;
        f[8 * t + 0] = __uint_as_float(and_or(lo, 0x0000Fu, kMagicBits));
        f[8 * t + 1] = __uint_as_float(and_or(lo, 0x000F0u, kMagicBits));
        f[8 * t + 2] = __uint_as_float(and_or(lo, 0x00F00u, kMagicBits));
        f[8 * t + 3] = __uint_as_float(and_or(lo, 0x0F000u, kMagicBits));
        f[8 * t + 4] = __uint_as_float(and_or(lo, 0xF0000u, kMagicBits));
        f[8 * t + 5] = __uint_as_float(and_or(hi, 0x000F0u, kMagicBits));
        f[8 * t + 6] = __uint_as_float(and_or(hi, 0x00F00u, kMagicBits));
        f[8 * t + 7] = __uint_as_float(and_or(hi, 0x0F000u, kMagicBits));
    }
}

template <>
__device__ __forceinline__ void unpack_seg<6>(const uint8_t *seg, float (&f)[PANEL])
{
    const uint32_t *w = reinterpret_cast<const uint32_t *>(seg);
    const uint32_t w0 = w[0], w1 = w[1], w2 = w[2];
    const uint32_t g[4] = {w0, __funnelshift_r(w0, w1, 24), __funnelshift_r(w1, w2, 16), w2 >> 8};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        f[4 * k + 0] = __uint_as_float(and_or(g[k], 0x0003Fu, kMagicBits));
        f[4 * k + 1] = __uint_as_float(and_or(g[k], 0x00FC0u, kMagicBits));
        f[4 * k + 2] = __uint_as_float(and_or(g[k], 0x3F000u, kMagicBits));
        f[4 * k + 3] = __uint_as_float(and_or(g[k] >> 12, 0x00FC0u, kMagicBits));
    }
}

// codes (times their position scale) of one row segment, as exact floats
template <int BITS>
__device__ __forceinline__ void load_codes(const uint8_t *seg, float (&f)[PANEL])
{
    unpack_seg<BITS>(seg, f);
#pragma unroll
    for (int p = 0; p < PANEL; p += 2) {
        const float2 r = fadd2(make_float2(f[p], f[p + 1]),
                               make_float2(-pos_bias(BITS, p), -pos_bias(BITS, p + 1)));
        f[p] = r.x;
        f[p + 1] = r.y;
    }
}

// codes of one row segment with the position scale removed (exact code values), for rows
// whose widths differ inside one head: fma(f, 1/s, -(2^23 / s + 2^(b-1))) is exact
template <int BITS>
__device__ __forceinline__ void load_codes_unscaled(const uint8_t *seg, float (&f)[PANEL])
{
    unpack_seg<BITS>(seg, f);
#pragma unroll
    for (int p = 0; p < PANEL; p += 2) {
        const float2 r = ffma2(make_float2(f[p], f[p + 1]),
                               make_float2(1.0f / pos_scale(BITS, p), 1.0f / pos_scale(BITS, p + 1)),
                               make_float2(-pos_bias(BITS, p) / pos_scale(BITS, p),
                                           -pos_bias(BITS, p + 1) / pos_scale(BITS, p + 1)));
        f[p] = r.x;
        f[p + 1] = r.y;
    }
}

// Per-key-row widths: a head's rows are stored 8-bit first, then 4-bit, then 6-bit; stored
// row p has this width and starts this many bytes into its panel.
__device__ __forceinline__ int row_width(int p, int n8, int n4) { return p < n8 ? 8 : p < n8 + n4 ? 4 : 6; }
__device__ __forceinline__ int row_seg_off(int p, int n8, int n4)
{
    return p < n8 ? 16 * p : p < n8 + n4 ? 16 * n8 + 8 * (p - n8) : 16 * n8 + 8 * n4 + 12 * (p - n8 - n4);
}

// ---------------------------------------------------------------- pack one row segment
// Input: raw bits of fma(x, 1, 2^23 + 2^(b-1)) results, i.e. 0x4B000000 + u.

template <int BITS>
__device__ __forceinline__ void pack_seg(const uint32_t (&u)[PANEL], uint8_t *seg);

template <>
__device__ __forceinline__ void pack_seg<8>(const uint32_t (&u)[PANEL], uint8_t *seg)
{
    uint32_t ws[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const uint32_t lo = __byte_perm(u[4 * t + 0], u[4 * t + 1], 0x0040u);
        const uint32_t hi = __byte_perm(u[4 * t + 2], u[4 * t + 3], 0x0040u);
        ws[t] = __byte_perm(lo, hi, 0x5410u);
    }
    *reinterpret_cast<uint4 *>(seg) = make_uint4(ws[0], ws[1], ws[2], ws[3]);
}

template <>
__device__ __forceinline__ void pack_seg<4>(const uint32_t (&u)[PANEL], uint8_t *seg)
{
    constexpr uint32_t K = kMagicBits * 0x11111111u;     // wraps mod 2^32
    uint32_t ws[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        uint32_t acc = u[8 * t] - K;
#pragma unroll
        for (int e = 1; e < 8; ++e) acc += u[8 * t + e] << (4 * e);
        ws[t] = acc;
    }
    *reinterpret_cast<uint2 *>(seg) = make_uint2(ws[0], ws[1]);
}

template <>
__device__ __forceinline__ void pack_seg<6>(const uint32_t (&u)[PANEL], uint8_t *seg)
{
    constexpr uint32_t K = kMagicBits * (1u + 64u + 4096u + 262144u);
    uint32_t g[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        g[k] = (u[4 * k] - K) + (u[4 * k + 1] << 6) + (u[4 * k + 2] << 12) + (u[4 * k + 3] << 18);
    uint32_t *w = reinterpret_cast<uint32_t *>(seg);
    w[0] = g[0] | (g[1] << 24);
    w[1] = (g[1] >> 8) | (g[2] << 16);
    w[2] = (g[2] >> 16) | (g[3] << 8);
}

// ---------------------------------------------------------------- warp reductions

// Reduce-scatter of NV values over the lanes that differ in the bits OFF0, OFF0/2, ...
// (NSTEP halvings).  Afterwards a[0 .. NV >> NSTEP) hold the lane's share: original
// index sum_s (lane & (OFF0 >> s) ? (NV >> s) / 2 : 0) + (0 .. NV >> NSTEP).
template <int NV, int NSTEP, int OFF0, bool MAX>
__device__ __forceinline__ void reduce_scatter(float (&a)[NV], int lane)
{
#pragma unroll
    for (int s = 0; s < NSTEP; ++s) {
        const int o = OFF0 >> s;
        const int h = (NV >> s) / 2;
        const bool upper = (lane & o) != 0;
        float keep[NV / 2], recv[NV / 2];
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = upper ? a[i] : a[i + h];
            keep[i] = upper ? a[i + h] : a[i];
            recv[i] = __shfl_xor_sync(0xffffffffu, send, o);
        }
#pragma unroll
        for (int i = 0; i < h; i += 2) {
            if (MAX || i + 1 >= h) {
                a[i] = MAX ? fmaxf(keep[i], recv[i]) : keep[i] + recv[i];
                if (i + 1 < h) a[i + 1] = fmaxf(keep[i + 1], recv[i + 1]);
            } else {                        // two sums in one f32x2 add (the same IEEE adds)
                const float2 t = fadd2(make_float2(keep[i], keep[i + 1]), make_float2(recv[i], recv[i + 1]));
                a[i] = t.x;
                a[i + 1] = t.y;
            }
        }
    }
}

// ---------------------------------------------------------------- thread layout

template <int ROWS>
struct Layout {
    static_assert(ROWS == 4 || ROWS == 8, "ROWS must be 4 or 8");
    static constexpr int LP = DK / ROWS;          // lanes sharing a panel
    static constexpr int PW = 32 / LP;            // panels per warp
    static constexpr int NWARP = NPANEL / PW;
    static constexpr int NT = NWARP * 32;         // threads per state
    static constexpr int LOG_LP = LP == 32 ? 5 : 4;
};

template <int ROWS>
struct TileIdx {
    int lane, panel, rl, sw;
    __device__ __forceinline__ explicit TileIdx(int tid)
    {
        using L = Layout<ROWS>;
        lane = tid & 31;
        const int warp = tid >> 5;
        panel = warp * L::PW + lane / L::LP;
        rl = lane % L::LP;
        sw = (L::PW == 2) ? (lane / L::LP) : 0;   // bank-conflict swizzle of the row order
    }
    __device__ __forceinline__ int row(int m) const { return rl + Layout<ROWS>::LP * (m ^ sw); }
};

}  // namespace stepq
