// stepq_decode.cu -- the fused decode step of the quantized gated Delta-rule layer (sm_100a).
//
// Per (request b, value head h) state, one pass (STEPQuant summary, "Method": update the
// reconstructed state in floating point, compute the output, then quantize for storage;
// "Paper Explained", "The mechanism: rewriting state with the delta rule"):
//   S'_ij = alpha_i r_i c_j Q_ij            dequantize + fade
//   u_j   = sum_i S'_ij k_i                 predict (what the key currently retrieves)
//   d_j   = beta (v_j - u_j)                write strength times the difference
//   S_ij  = S'_ij + k_i d_j                 Delta write
//   y_j   = sum_i S_ij q_i                  readout from the updated, unquantized state
//   c_j   = sqrt(max_i |S_ij|),  r_i = max_j (|S_ij| / c_j) / qmax      clip-free refit
//   Q_ij  = round-half-even(S_ij / (r_i c_j)), repacked in place
//
// Arithmetic: with rho_i = alpha_i r_i, both column dot products run on the integer codes
// with per-row weights (u_j = c_j sum_i Q_ij rho_i k_i, y'_j = c_j sum_i Q_ij rho_i q_i,
// y_j = y'_j + (k.q) d_j), and the updated state is kept column-scaled:
// S_ij = c_j T_ij with T_ij = rho_i Q_ij + k_i (d_j / c_j).  The refit then needs
// max_i |T_ij|, the new column factor, and P_ij = T_ij (c_j / c_new_j) = S_ij / c_new_j.
//
// Threads: 256 per state.  Warp w owns the 16-column panel w; lane l holds rows l + 32 m
// (m = 0..3) of it: 64 state values in registers.  Column sums and maxima reduce over the
// warp's lanes.  Row maxima over the 8 panels go through shared memory, where thread t
// (t < 128) finalizes row t (r_t and 1/r_t) while threads 128..255 build the per-row
// weights of the next state, so every row-wise quantity is computed once.  Row weights
// are stored as duplicated pairs, the operand form of the packed f32x2 instructions.
//
// Data movement: persistent CTAs; items are dealt round-robin in head-major order and the
// heads are visited grouped by bit width, so the CTAs resident at a time share one code
// path.  Thread 0 bulk-copies the packed head block and q, k, v (and the KDA gate) of item
// i+2 into a 4-stage shared-memory ring while the CTA computes item i (full barriers:
// mbarrier transaction counts; empty barriers: one arrival per warp once its stores have
// read the stage).  After the refit each warp bulk-stores its panel and its slice of c
// from the stage (warp 0 also r).  Each state is read from HBM once and written once.
#include <cfloat>
#include <cstdint>
#include <type_traits>
#include <cuda_fp16.h>

#include "stepq_internal.h"
#include "stepq_tile.cuh"

namespace stepq {

namespace {

constexpr int kStages = 4;
constexpr int kIoBytes = 512;       // stage room for one 128-vector input (fp32 or bf16)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 4;            // rows per thread
constexpr unsigned kFull = 0xffffffffu;
// Stage of the ring: room for the largest quantized head block (8-bit codes + r + c; a head
// with per-key-row widths is never larger), then q, k, v and, for KDA, the gate vector.
constexpr int kBlkCap = block_bytes(8);
template <int GATE>
__host__ __device__ constexpr int stage_bytes_of()
{
    return (kBlkCap + (GATE == STEPQ_GATE_KDA ? 4 : 3) * kIoBytes + 127) / 128 * 128;
}

struct StageMeta {
    long long dst;                  // byte offset of the head block in the pool
    int valid;
    int bits;                       // 4, 6, 8, or 0: per-key-row widths
    int head;
};

struct DecodeArgs {
    uint8_t *pool;
    long long slot_stride;
    const long long *head_off;
    const uint8_t *head_bits;
    const int32_t *head_order;      // processing order of the heads (grouped by bit width)
    int num_slots, H, Hk, group;
    int nh4, nh6, nh8;              // heads of width 4, 6 and 8 (visited in that order, then the
                                    // heads with per-key-row widths)
    // heads with per-key-row widths (width 0): block bytes, rows of width 8 and 4 (stored
    // first, in that order; the rest are 6-bit), padded panel bytes, stored row -> key row
    const int32_t *head_blk;
    const uint8_t *row_n8, *row_n4;
    const int32_t *row_pb;
    const uint8_t *row_perm;
    int Hq;                         // quantized heads: the first Hq entries of head_order
    const float *impact;            // [H, d_k] normalized row-impact weights (impact fit), or null
    const int32_t *slot_ids;
    int n;
    int step_b, step_h;             // gridDim.x in head-major items = step_h * n + step_b
    const void *q, *k, *v, *alpha, *beta;
    float *y;
    int *flag;
};

// Shared memory besides the ring.
struct Scratch {
    float rp[NPANEL * DK];          // row maxima of |P|: [panel][row] (conflict-free stores and loads)
    float4 wlo[DK];                 // per row {rho k, rho k, rho q, rho q}  (lanes 0..15)
    float4 whi[DK];                 // per row {rho q, rho q, rho k, rho k}  (lanes 16..31)
    float4 wrk[DK];                 // per row {rho, rho, k, k}
    float2 ir[DK];                  // per row {1/r, 1/r}
    float4 fit[DK];                 // impact fit, per row {1/r, 1/r, w r^2, w r^2}
    float xd[NPANEL * PANEL];       // d_j / c'_j per column
    float xg[NPANEL * PANEL];       // c'_j / c_new_j per column
    float kqw[4];                   // partial k.q of the next state (warps 4..7)
    float invpos[3][PANEL];         // 1 / position scale of the unpacked field (bits 4, 6, 8)
    long long hoff[kMaxHeads];      // head block offsets inside a slot
    int32_t hord[kMaxHeads];        // head processing order
    uint8_t hbits[kMaxHeads];       // head widths
    uint8_t hkey[kMaxHeads];        // key head of each value head (h / group)
    // heads with per-key-row widths (pools that have such heads): padded panel bytes and the
    // counts of 8-bit and 4-bit rows
    int32_t rpb[kMaxHeads];
    uint8_t rn8[kMaxHeads], rn4[kMaxHeads];
    StageMeta meta[kStages];
    int prod_b, prod_h;             // producer cursor
    uint64_t full[kStages];
    uint64_t empty[kStages];
};

// 1 / (power-of-two scale of the unpacked field) by bit width and column in the panel
__constant__ float kInvPos[3][PANEL];

// Item cursor in head-major order (index = h * n + b), stepping by the grid size.
struct Cursor {
    int b, h;
    __device__ __forceinline__ void advance(const DecodeArgs &a)
    {
        b += a.step_b;
        h += a.step_h;
        if (b >= a.n) { b -= a.n; ++h; }
    }
};

// Per-row weights of a state held in a stage, built by thread t (128 <= t < 256) for row
// t - 128, and the share of k.q of warps 4..7.
template <int GATE, typename TIn, bool ROWS>
__device__ __forceinline__ void row_table(const uint8_t *stage, const DecodeArgs &a, int bits, int head,
                                          float alpha_s, Scratch &sc, int t)
{
    const int i = t - 128;                          // stored row (the key row unless bits == 0)
    const bool rows = ROWS && bits == 0;            // heads with per-key-row widths exist only in ROWS pools
    const float *r = reinterpret_cast<const float *>(stage + (rows ? NPANEL * sc.rpb[head] : codes_bytes(bits)));
    const int key = rows ? int(a.row_perm[head * DK + i]) : i;
    const TIn *qs = reinterpret_cast<const TIn *>(stage + kBlkCap);
    const TIn *ks = reinterpret_cast<const TIn *>(stage + kBlkCap + kIoBytes);
    const TIn *as = reinterpret_cast<const TIn *>(stage + kBlkCap + 3 * kIoBytes);
    const float al = (GATE == STEPQ_GATE_KDA) ? to_f32(as[key]) : alpha_s;
    const float rho = al * r[i];
    const float k = to_f32(ks[key]);
    const float q = to_f32(qs[key]);
    const float rk = rho * k, rq = rho * q;
    sc.wlo[i] = make_float4(rk, rk, rq, rq);
    sc.whi[i] = make_float4(rq, rq, rk, rk);
    sc.wrk[i] = make_float4(rho, rho, k, k);
    float kq = k * q;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) kq += __shfl_xor_sync(kFull, kq, o);
    if ((t & 31) == 0) sc.kqw[(t >> 5) - 4] = kq;
}

// Lane 0 of each warp, after issuing its stores of item i: close them as one bulk group, then
// wait until the warp's stores of item i-1 have read their stage and release that stage to
// the producer (one arrival per warp on its empty barrier).
__device__ __forceinline__ void retire_stores(Scratch &sc, int i)
{
    bulk_commit();
    if (i >= 1) {
        bulk_wait_read<1>();
        mbar_arrive(&sc.empty[(i - 1) % kStages]);
    }
}

// One state: the register tile through the row-maxima exchange, the row finalization /
// next row table, then quantization, packing and the per-warp stores.  Returns false on
// every thread when some thread saw a failed wait.
template <int GATE, typename TIn, int BITS, bool ROWS>
__device__ __forceinline__ bool refit_impact(float (&T)[kRows][PANEL], uint8_t *stages, int i, bool has_next,
                                             const DecodeArgs &a, Scratch &sc, const TileIdx<4> &ix, int tid, int h,
                                             float cprime, TIn alpha_next_raw, bool ok, float *r_io, float *c_io,
                                             uint8_t *codes);

// In the impact-fit instantiations the clip-free fit after the early return to refit_impact is
// never reached; the front end reports its loops as unreachable there.
#pragma nv_diagnostic push
#pragma nv_diag_suppress 128
template <int GATE, typename TIn, int BITS, bool IMPACT, bool ROWS>
__device__ __forceinline__ bool decode_item(uint8_t *stages, int i, bool has_next, const DecodeArgs &a, Scratch &sc,
                                            const TileIdx<4> &ix, int tid, int bh, float beta, float kq,
                                            TIn alpha_next_raw, bool ok)
{
    uint8_t *stage = stages + (i % kStages) * stage_bytes_of<GATE>();
    // BITS == 0: per-key-row widths (rows stored 8-bit, 4-bit, 6-bit; codes unscaled)
    constexpr int QM = BITS ? qmax_of(BITS) : 1;
    constexpr float MAG = kTwo23 + float(1 << ((BITS ? BITS : 1) - 1));
    constexpr int BI = BITS == 4 ? 0 : BITS == 6 ? 1 : 2;
    const int lane = ix.lane;
    const int panel = ix.panel;
    const bool upper = (lane & 16) != 0;            // lanes holding the q-weighted sums first
    const int col = lane & 15;                      // the column this lane finalizes
    const int head = sc.meta[i % kStages].head;
    int n8 = 0, n4 = 0, pb = panel_bytes(BITS ? BITS : 4);
    if constexpr (BITS == 0) {
        n8 = sc.rn8[head];
        n4 = sc.rn4[head];
        pb = sc.rpb[head];
    }
    const int cbytes = BITS ? codes_bytes(BITS) : 8 * pb;

    uint8_t *codes = stage;
    float *r_io = reinterpret_cast<float *>(stage + cbytes);
    float *c_io = r_io + DK;
    const TIn *vs = reinterpret_cast<const TIn *>(stage + kBlkCap + 2 * kIoBytes);

    // ---- codes of the thread's 4 rows x 16 columns (times their position scale), exact floats
    float T[kRows][PANEL];
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
        if constexpr (BITS == 0) {
            const int p = ix.row(m);
            const uint8_t *seg = codes + panel * pb + row_seg_off(p, n8, n4);
            const int wdt = row_width(p, n8, n4);
            if (wdt == 8)
                load_codes_unscaled<8>(seg, T[m]);
            else if (wdt == 4)
                load_codes_unscaled<4>(seg, T[m]);
            else
                load_codes_unscaled<6>(seg, T[m]);
        } else {
            load_codes<BITS>(codes + panel * panel_bytes(BITS) + ix.row(m) * seg_bytes(BITS), T[m]);
        }
    }

    // A zero column factor means a zero column whatever its codes (a fresh pool holds
    // nonzero codes under zero scales): clear those codes.  Warp-uniform and rare.
    const float cj = c_io[panel * PANEL + col];
    if (__any_sync(kFull, cj == 0.0f)) {
#pragma unroll
        for (int j = 0; j < PANEL; ++j) {
            const float z = c_io[panel * PANEL + j] == 0.0f ? 0.0f : 1.0f;
#pragma unroll
            for (int m = 0; m < kRows; ++m) T[m][j] *= z;
        }
    }
    // column factor of the scaled codes (a zero column behaves as c = 1: S = T = k d)
    const float cprime = (cj == 0.0f ? 1.0f : cj) * (BITS ? sc.invpos[BI][col] : 1.0f);

    // ---- column dot products over the thread's rows (column pairs, f32x2), then over the
    // warp: lane bit 4 first (select-free: the partner's second sum is this lane's first
    // quantity), then bits 3..0.  Lanes 0..15 end with u_col, lanes 16..31 with y'_col.
    const float4 *wt = upper ? sc.whi : sc.wlo;
    float4 w[kRows];
#pragma unroll
    for (int m = 0; m < kRows; ++m) w[m] = wt[ix.row(m)];
    float A[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 2) {
        float2 s1 = fmul2(make_float2(T[0][j], T[0][j + 1]), make_float2(w[0].x, w[0].y));
        float2 s2 = fmul2(make_float2(T[0][j], T[0][j + 1]), make_float2(w[0].z, w[0].w));
#pragma unroll
        for (int m = 1; m < kRows; ++m) {
            s1 = ffma2(make_float2(T[m][j], T[m][j + 1]), make_float2(w[m].x, w[m].y), s1);
            s2 = ffma2(make_float2(T[m][j], T[m][j + 1]), make_float2(w[m].z, w[m].w), s2);
        }
        const float2 t = fadd2(s1, make_float2(__shfl_xor_sync(kFull, s2.x, 16), __shfl_xor_sync(kFull, s2.y, 16)));
        A[j] = t.x;
        A[j + 1] = t.y;
    }
    reduce_scatter<PANEL, 4, 8, false>(A, lane);

    // d_j = beta (v_j - u_j) (lanes 0..15); y_j = y'_j + (k.q) d_j (lanes 16..31)
    const float val = cprime * A[0];
    const float delta = beta * (to_f32(vs[panel * PANEL + col]) - val);
    const float dpair = __shfl_xor_sync(kFull, delta, 16);
    st_global_if(upper, a.y + (long long)bh * DV + panel * PANEL + col, fmaf(dpair, kq, val));
    st_shared_if(!upper, sc.xd + panel * PANEL + col, div_refined(delta, cprime));
    __syncwarp();
    float dd[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(sc.xd + panel * PANEL + j);
        dd[j] = t.x; dd[j + 1] = t.y; dd[j + 2] = t.z; dd[j + 3] = t.w;
    }

    // ---- T_ij = rho_i Q_ij + k_i d'_j (the updated state is c'_j T_ij); column maxima of |T|
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
        const float4 rk = sc.wrk[ix.row(m)];
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            float2 t = fmul2(make_float2(T[m][j], T[m][j + 1]), make_float2(rk.x, rk.y));
            t = ffma2(make_float2(rk.z, rk.w), make_float2(dd[j], dd[j + 1]), t);
            T[m][j] = t.x;
            T[m][j + 1] = t.y;
        }
    }
    if constexpr (IMPACT && BITS != 0)          // heads with per-row widths keep the clip-free fit
        return refit_impact<GATE, TIn, BITS, ROWS>(T, stages, i, has_next, a, sc, ix, tid, head, cprime,
                                             alpha_next_raw, ok, r_io, c_io, codes);
    // column maxima: over the thread's rows, then a warp-wide max per column; the 16
    // results go through shared memory (the d' buffer, already read) to the column lanes
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        float cm[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            cm[e] = warp_absmax(fmaxf(absmax3(T[0][j + e], T[1][j + e], T[2][j + e]), fabsf(T[3][j + e])));
        st_shared_v4_if(lane == 0, sc.xd + panel * PANEL + j, make_float4(cm[0], cm[1], cm[2], cm[3]));
    }
    __syncwarp();
    const float tmax = sc.xd[panel * PANEL + col];

    // c_new = sqrt(max_i |S_ij|); the scaled state divides by it: g_j = c'_j / c_new_j
    const float cnew = sqrt_refined(cprime * tmax);
    const float g = cnew > 0.0f ? div_refined(cprime, cnew) : 0.0f;
    st_shared_if(!upper, c_io + panel * PANEL + col, cnew);
    st_shared_if(!upper, sc.xg + panel * PANEL + col, g);
    __syncwarp();
    float gg[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(sc.xg + panel * PANEL + j);
        gg[j] = t.x; gg[j + 1] = t.y; gg[j + 2] = t.z; gg[j + 3] = t.w;
    }
    // P_ij = S_ij / c_new_j and the thread's row maxima of |P| (panel partials)
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            const float2 p = fmul2(make_float2(T[m][j], T[m][j + 1]), make_float2(gg[j], gg[j + 1]));
            T[m][j] = p.x;
            T[m][j + 1] = p.y;
        }
        float mx = absmax3(T[m][0], T[m][1], T[m][2]);
#pragma unroll
        for (int j = 3; j < PANEL - 1; j += 2) mx = absmax3(mx, T[m][j], T[m][j + 1]);
        mx = fmaxf(mx, fabsf(T[m][PANEL - 1]));
        sc.rp[panel * DK + ix.row(m)] = mx;
    }
    if (__syncthreads_or(!ok)) return false;

    // ---- threads 0..127: r_t = max_j |P_tj| / qmax and 1 / r_t for row t;
    //      threads 128..255: the next state's row weights
    bool tiny = false;
    if (tid < DK) {
        const float *rpt = sc.rp + tid;
        const float mr = fmaxf(max3(rpt[0], rpt[DK], rpt[2 * DK]),
                               max3(max3(rpt[3 * DK], rpt[4 * DK], rpt[5 * DK]), rpt[6 * DK], rpt[7 * DK]));
        float r;
        if constexpr (BITS == 0) {
            const int wdt = row_width(tid, n8, n4);
            r = div_refined(mr, float(qmax_of(wdt)));
            const float ir = r >= FLT_MIN ? rcp_refined(r) : 0.0f;
            const float mag = kTwo23 + float(1 << (wdt - 1));
            sc.fit[tid] = make_float4(ir, ir, mag, mag);
        } else {
            r = div_const<QM>(mr);
            const float ir = r >= FLT_MIN ? rcp_refined(r) : 0.0f;
            sc.ir[tid] = make_float2(ir, ir);
        }
        r_io[tid] = r;
        tiny = r > 0.0f && r < FLT_MIN;
    } else if (has_next && sc.meta[(i + 1) % kStages].valid) {
        row_table<GATE, TIn, ROWS>(stages + ((i + 1) % kStages) * stage_bytes_of<GATE>(), a, sc.meta[(i + 1) % kStages].bits,
                             sc.meta[(i + 1) % kStages].head, to_f32(alpha_next_raw), sc, tid);
    }
    const bool any_tiny = __syncthreads_or(tiny);

    // ---- codes = round-half-even(P_ij / r_i): fma(P, 1/r, 2^23 + 2^(b-1)) rounds to the
    // nearest integer, ties to even, leaving the offset-binary code in the low mantissa bits.
    // The block-uniform any_tiny picks one of two copies of the loop, so the common copy has
    // no per-row test.
    auto quantize_pack = [&](auto tiny_rows) {
#pragma unroll
        for (int m = 0; m < kRows; ++m) {
            const int row = ix.row(m);
            float2 ir, mag2 = make_float2(MAG, MAG);
            if constexpr (BITS == 0) {
                const float4 f = sc.fit[row];
                ir = make_float2(f.x, f.y);
                mag2 = make_float2(f.z, f.w);
            } else {
                ir = sc.ir[row];
            }
            uint32_t u[PANEL];
#pragma unroll
            for (int j = 0; j < PANEL; j += 2) {
                const float2 f = ffma2(make_float2(T[m][j], T[m][j + 1]), ir, mag2);
                u[j] = __float_as_uint(f.x);
                u[j + 1] = __float_as_uint(f.y);
            }
            if constexpr (decltype(tiny_rows)::value) {
                // subnormal row factor: 1/r overflows; scale P and r by 2^64 (exact: |P| <= qmax r)
                const float r = r_io[row];
                if (r > 0.0f && r < FLT_MIN) {
                    const float irs = rcp_refined(r * 0x1p64f);
#pragma unroll
                    for (int j = 0; j < PANEL; ++j) u[j] = __float_as_uint(fmaf(T[m][j] * 0x1p64f, irs, mag2.x));
                }
            }
            if constexpr (BITS == 0) {
                uint8_t *seg = codes + panel * pb + row_seg_off(row, n8, n4);
                const int wdt = row_width(row, n8, n4);
                if (wdt == 8)
                    pack_seg<8>(u, seg);
                else if (wdt == 4)
                    pack_seg<4>(u, seg);
                else
                    pack_seg<6>(u, seg);
            } else {
                pack_seg<BITS>(u, codes + panel * panel_bytes(BITS) + row * seg_bytes(BITS));
            }
        }
    };
    if (any_tiny)
        quantize_pack(std::true_type{});
    else
        quantize_pack(std::false_type{});
    // each warp stores its panel of codes and its slice of c (warp 0 also r)
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        uint8_t *dst = a.pool + sc.meta[i % kStages].dst;
        bulk_s2g(dst + panel * pb, codes + panel * pb, uint32_t(pb));
        bulk_s2g(dst + cbytes + 4 * DK + 4 * PANEL * panel, c_io + PANEL * panel, 4 * PANEL);
        if (panel == 0) bulk_s2g(dst + cbytes, r_io, 4 * DK);
        retire_stores(sc, i);
    }
    return true;
}

#pragma nv_diagnostic pop

// Key-row-aware dual-axis fit with row-impact weights (STEPQuant summary, "Method" para 4):
// on entry T_ij = S_ij / c'_j.  r_i = sqrt(max_j |S_ij| / w_i); c0_j = max_i |S_ij / r_i| / qmax;
// Q0 = nearest levels of S / (r c0); c_j = sum_i w_i r_i Q0_ij S_ij / sum_i w_i r_i^2 Q0_ij^2
// (c0_j when a sum is not positive); codes = nearest levels of S / (r c), clipped.  With
// P_ij = S_ij / r_i the sums are sum (w r^2) Q0 P and sum (w r^2) Q0^2, reduced over the warp
// like the column dot products.
template <int GATE, typename TIn, int BITS, bool ROWS>
__device__ __forceinline__ bool refit_impact(float (&T)[kRows][PANEL], uint8_t *stages, int i, bool has_next,
                                             const DecodeArgs &a, Scratch &sc, const TileIdx<4> &ix, int tid, int h,
                                             float cprime, TIn alpha_next_raw, bool ok, float *r_io, float *c_io,
                                             uint8_t *codes)
{
    constexpr int QM = qmax_of(BITS);
    constexpr float MAG = kTwo23 + float(1 << (BITS - 1));
    const int lane = ix.lane;
    const int panel = ix.panel;
    const bool upper = (lane & 16) != 0;
    const int col = lane & 15;
    float *cbuf = sc.xg + panel * PANEL;            // one value per column of the panel

    // S_ij = c'_j T_ij, and the thread's row maxima of |S| (panel partials)
    st_shared_if(!upper, cbuf + col, cprime);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 cp = *reinterpret_cast<const float4 *>(cbuf + j);
#pragma unroll
        for (int m = 0; m < kRows; ++m) {
            const float2 x = fmul2(make_float2(T[m][j], T[m][j + 1]), make_float2(cp.x, cp.y));
            const float2 z = fmul2(make_float2(T[m][j + 2], T[m][j + 3]), make_float2(cp.z, cp.w));
            T[m][j] = x.x; T[m][j + 1] = x.y; T[m][j + 2] = z.x; T[m][j + 3] = z.y;
        }
    }
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
        float mx = absmax3(T[m][0], T[m][1], T[m][2]);
#pragma unroll
        for (int j = 3; j < PANEL - 1; j += 2) mx = absmax3(mx, T[m][j], T[m][j + 1]);
        mx = fmaxf(mx, fabsf(T[m][PANEL - 1]));
        sc.rp[panel * DK + ix.row(m)] = mx;
    }
    if (__syncthreads_or(!ok)) return false;

    // ---- threads 0..127: r, 1/r and w r^2 of row tid (IEEE sqrt and divide; r is normal);
    //      threads 128..255: the next state's row weights
    if (tid < DK) {
        const float *rpt = sc.rp + tid;
        const float mr = fmaxf(max3(rpt[0], rpt[DK], rpt[2 * DK]),
                               max3(max3(rpt[3 * DK], rpt[4 * DK], rpt[5 * DK]), rpt[6 * DK], rpt[7 * DK]));
        const float w = a.impact[h * DK + tid];
        const float r = __fsqrt_rn(__fdiv_rn(mr, w));
        r_io[tid] = r;
        const float ir = r > 0.0f ? __frcp_rn(r) : 0.0f;
        const float wr2 = w * r * r;
        sc.fit[tid] = make_float4(ir, ir, wr2, wr2);
        fence_proxy_async_smem();                  // r is bulk-stored from the stage by warp 0
    } else if (has_next && sc.meta[(i + 1) % kStages].valid) {
        row_table<GATE, TIn, ROWS>(stages + ((i + 1) % kStages) * stage_bytes_of<GATE>(), a, sc.meta[(i + 1) % kStages].bits,
                             sc.meta[(i + 1) % kStages].head, to_f32(alpha_next_raw), sc, tid);
    }
    __syncthreads();

    // ---- P_ij = S_ij / r_i; column maxima of |P| give c0 = max / qmax
    float2 wr[kRows];
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
        const float4 f = sc.fit[ix.row(m)];
        wr[m] = make_float2(f.z, f.w);
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            const float2 p = fmul2(make_float2(T[m][j], T[m][j + 1]), make_float2(f.x, f.y));
            T[m][j] = p.x;
            T[m][j + 1] = p.y;
        }
    }
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        float cm[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            cm[e] = warp_absmax(fmaxf(absmax3(T[0][j + e], T[1][j + e], T[2][j + e]), fabsf(T[3][j + e])));
        st_shared_v4_if(lane == 0, sc.xd + panel * PANEL + j, make_float4(cm[0], cm[1], cm[2], cm[3]));
    }
    __syncwarp();
    const float c0 = div_const<QM>(sc.xd[panel * PANEL + col]);
    st_shared_if(!upper, cbuf + col, c0 > 0.0f ? rcp_refined(c0) : 0.0f);
    __syncwarp();

    // ---- codes Q0 under c0 and the weighted least-squares sums of each column: lanes 0..15
    // keep the numerators after the first reduce step, lanes 16..31 the denominators
    float A[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 2) {
        const float2 ic = *reinterpret_cast<const float2 *>(cbuf + j);
        float2 sn = make_float2(0.0f, 0.0f), sd = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int m = 0; m < kRows; ++m) {
            const float2 p = make_float2(T[m][j], T[m][j + 1]);
            const float2 q0 = fadd2(ffma2(p, ic, make_float2(MAG, MAG)), make_float2(-MAG, -MAG));
            const float2 z = fmul2(q0, wr[m]);
            sn = ffma2(z, p, sn);
            sd = ffma2(z, q0, sd);
        }
        A[j] = (upper ? sd.x : sn.x) + __shfl_xor_sync(kFull, upper ? sn.x : sd.x, 16);
        A[j + 1] = (upper ? sd.y : sn.y) + __shfl_xor_sync(kFull, upper ? sn.y : sd.y, 16);
    }
    reduce_scatter<PANEL, 4, 8, false>(A, lane);
    const float other = __shfl_xor_sync(kFull, A[0], 16);
    const float num = upper ? other : A[0], den = upper ? A[0] : other;
    const float c1 = (num > 0.0f && den > 0.0f) ? div_refined(num, den) : c0;
    st_shared_if(!upper, c_io + panel * PANEL + col, c1);
    st_shared_if(!upper, cbuf + col, c1 > 0.0f ? rcp_refined(c1) : 0.0f);
    __syncwarp();
    float icl[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 t4 = *reinterpret_cast<const float4 *>(cbuf + j);
        icl[j] = t4.x; icl[j + 1] = t4.y; icl[j + 2] = t4.z; icl[j + 3] = t4.w;
    }

    // ---- codes = nearest levels of P / c, clipped to [-qmax, qmax]
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
        uint32_t u[PANEL];
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            const float2 f = ffma2(make_float2(T[m][j], T[m][j + 1]), make_float2(icl[j], icl[j + 1]),
                                   make_float2(MAG, MAG));
            u[j] = __float_as_uint(fminf(fmaxf(f.x, MAG - float(QM)), MAG + float(QM)));
            u[j + 1] = __float_as_uint(fminf(fmaxf(f.y, MAG - float(QM)), MAG + float(QM)));
        }
        pack_seg<BITS>(u, codes + panel * panel_bytes(BITS) + ix.row(m) * seg_bytes(BITS));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        uint8_t *dst = a.pool + sc.meta[i % kStages].dst;
        bulk_s2g(dst + panel * panel_bytes(BITS), codes + panel * panel_bytes(BITS), panel_bytes(BITS));
        bulk_s2g(dst + codes_bytes(BITS) + 4 * DK + 4 * PANEL * panel, c_io + PANEL * panel, 4 * PANEL);
        if (panel == 0) bulk_s2g(dst + codes_bytes(BITS), r_io, 4 * DK);
        retire_stores(sc, i);
    }
    return true;
}

// Per-CTA state of the item loop.  The loop runs in three pieces, one per bit width
// (the heads are visited grouped by width), so each piece is compiled for one width.
template <int GATE, typename TIn, bool IMPACT, bool ROWS>
struct ItemLoop {
    const DecodeArgs &a;
    Scratch &sc;
    uint8_t *stages;
    TileIdx<4> ix;
    int tid, lane, count;
    Cursor cur;
    int bh_cur;                         // b * H + h of the current item
    float beta_cur;
    bool ok;
    int slot_next;                      // producer: prefetched slot id of the next item to issue

    __device__ __forceinline__ ItemLoop(const DecodeArgs &a_, Scratch &sc_, uint8_t *stages_, int tid_, int count_)
        : a(a_), sc(sc_), stages(stages_), ix(tid_), tid(tid_), lane(tid_ & 31), count(count_), ok(true), slot_next(0)
    {
    }

    // producer (thread 0): bulk-copy item j's inputs into stage j % kStages
    __device__ __forceinline__ void issue(int j)
    {
        constexpr int esz = sizeof(TIn);
        const int st = j % kStages;
        const int slot = slot_next;
        Cursor pc = {sc.prod_b, sc.prod_h};
        const int b = pc.b, h = sc.hord[pc.h], g = sc.hkey[h];
        pc.advance(a);
        sc.prod_b = pc.b;
        sc.prod_h = pc.h;
        if (j + 1 < count) slot_next = __ldg(a.slot_ids + pc.b);
        uint8_t *stage = stages + st * stage_bytes_of<GATE>();
        StageMeta &mt = sc.meta[st];
        if (slot < 0 || slot >= a.num_slots) {
            mt.valid = 0;
            atomicOr(a.flag, STEPQ_FLAG_BAD_SLOT);
            mbar_arrive(&sc.full[st]);
        } else {
            const int bits = sc.hbits[h];
            const uint32_t bb = (ROWS && bits == 0) ? uint32_t(NPANEL * sc.rpb[h] + 4 * DK + 4 * DV)
                                                    : uint32_t(block_bytes(bits));
            const long long bh = (long long)b * a.H + h;
            const long long kqrow = (long long)b * a.Hk + g;
            mt.valid = 1;
            mt.bits = bits;
            mt.head = h;
            mt.dst = (long long)slot * a.slot_stride + sc.hoff[h];
            const uint32_t io = DK * esz;
            mbar_arrive_expect_tx(&sc.full[st], bb + 3 * io + (GATE == STEPQ_GATE_KDA ? io : 0u));
            bulk_g2s(stage, a.pool + mt.dst, bb, &sc.full[st]);
            bulk_g2s(stage + kBlkCap, static_cast<const uint8_t *>(a.q) + kqrow * io, io, &sc.full[st]);
            bulk_g2s(stage + kBlkCap + kIoBytes, static_cast<const uint8_t *>(a.k) + kqrow * io, io, &sc.full[st]);
            bulk_g2s(stage + kBlkCap + 2 * kIoBytes, static_cast<const uint8_t *>(a.v) + bh * io, io, &sc.full[st]);
            if (GATE == STEPQ_GATE_KDA)
                bulk_g2s(stage + kBlkCap + 3 * kIoBytes, static_cast<const uint8_t *>(a.alpha) + bh * io, io,
                         &sc.full[st]);
        }
    }

    // Items i .. i_end - 1, all of width BITS (or skipped: bad slot).  Returns false (with
    // i at the item) when a wait gave up.
    template <int BITS>
    __device__ __forceinline__ bool run(int &i, int i_end)
    {
        const TIn *alpha_g = static_cast<const TIn *>(a.alpha);
        const TIn *beta_g = static_cast<const TIn *>(a.beta);
        for (; i < i_end; ++i) {
            const int st = i % kStages;
            if (tid == 0 && i + 2 < count) {
                if (i + 2 >= kStages)                // stage (i+2)%4 last held item i-2
                    ok &= mbar_wait_bounded(&sc.empty[(i + 2) % kStages], uint32_t((i - 2) / kStages) & 1u);
                issue(i + 2);
            }
            // next item: cursor, scalar gates, its stage (waited for before its row table is built)
            Cursor nxt = cur;
            nxt.advance(a);
            const bool has_next = i + 1 < count;
            const int bh_next = has_next ? nxt.b * a.H + sc.hord[nxt.h] : 0;
            TIn beta_raw = TIn(0), alpha_raw = TIn(0);            // converted when used
            if (has_next) {
                beta_raw = beta_g[bh_next];
                if (GATE == STEPQ_GATE_GDN) alpha_raw = alpha_g[bh_next];
            }
            const float4 kqv = *reinterpret_cast<const float4 *>(sc.kqw);
            const float kq = (kqv.x + kqv.y) + (kqv.z + kqv.w);
            const int valid = sc.meta[st].valid;
            // one thread waits for the next item's stage: its copies become visible to that
            // thread, and the block barrier that follows (barrier 1 of this item, or the one
            // of an empty item) orders every other thread's reads of the stage after the wait
            if (has_next && tid == DK)
                ok &= mbar_wait_bounded(&sc.full[(i + 1) % kStages], uint32_t((i + 1) / kStages) & 1u);
            bool alive;
            if (!valid) {
                alive = !__syncthreads_or(!ok);
                if (alive) {
                    const StageMeta mn = sc.meta[(i + 1) % kStages];
                    if (has_next && mn.valid && tid >= DK)
                        row_table<GATE, TIn, ROWS>(stages + ((i + 1) % kStages) * stage_bytes_of<GATE>(), a, mn.bits, mn.head,
                                             to_f32(alpha_raw), sc, tid);
                    __syncthreads();
                    if (lane == 0) retire_stores(sc, i);     // an empty group keeps one group per item
                }
            } else {
                alive = decode_item<GATE, TIn, BITS, IMPACT, ROWS>(stages, i, has_next, a, sc, ix, tid, bh_cur, beta_cur, kq,
                                                     alpha_raw, ok);
            }
            if (!alive) return false;
            cur = nxt;
            bh_cur = bh_next;
            beta_cur = to_f32(beta_raw);
        }
        return true;
    }
};

template <int GATE, typename TIn, bool IMPACT, bool ROWS>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecodeArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *stages = smem;
    Scratch &sc = *reinterpret_cast<Scratch *>(smem + kStages * stage_bytes_of<GATE>());

    const int tid = threadIdx.x;
    const long long total = (long long)a.n * a.Hq;
    const long long first = blockIdx.x;
    if (first >= total) return;
    const long long G = gridDim.x;
    const int count = int((total - first + G - 1) / G);
    // this CTA's items are first + k G; those with k < end4 are on 4-bit heads, then 6-bit
    auto class_end = [&](long long e) {
        return e > first ? int(min((long long)count, (e - first + G - 1) / G)) : 0;
    };
    const int end4 = class_end((long long)a.nh4 * a.n);
    const int end6 = class_end((long long)(a.nh4 + a.nh6) * a.n);
    const int end8 = class_end((long long)(a.nh4 + a.nh6 + a.nh8) * a.n);

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sc.full[s], 1);
            mbar_init(&sc.empty[s], kWarps);
        }
        fence_mbarrier_init();
    }
    if (tid < 3 * PANEL) sc.invpos[tid / PANEL][tid % PANEL] = kInvPos[tid / PANEL][tid % PANEL];
    for (int h = tid; h < a.H; h += kThreads) {
        sc.hoff[h] = a.head_off[h];
        sc.hord[h] = a.head_order[h];
        sc.hbits[h] = a.head_bits[h];
        sc.hkey[h] = uint8_t(h / a.group);
        if constexpr (ROWS) {
            sc.rpb[h] = a.row_pb[h];
            sc.rn8[h] = a.row_n8[h];
            sc.rn4[h] = a.row_n4[h];
        }
    }
    __syncthreads();
    // everything above reads only the pool's tables; the states, the inputs and y may still be
    // in use by the previous grid of the stream when this one was launched as its dependent
    grid_dependency_wait();
    // the next grid may launch now: its CTAs become resident only as this grid's CTAs exit
    if (tid == 0) grid_launch_dependents();

    ItemLoop<GATE, TIn, IMPACT, ROWS> L(a, sc, stages, tid, count);
    L.cur = {int(first % a.n), int(first / a.n)};
    if (tid == 0) {
        sc.prod_b = L.cur.b;
        sc.prod_h = L.cur.h;
        L.slot_next = __ldg(a.slot_ids + L.cur.b);
        L.issue(0);
        if (count > 1) L.issue(1);
    }

    // ---- prologue: the first state's row table
    const TIn *alpha_g = static_cast<const TIn *>(a.alpha);
    const TIn *beta_g = static_cast<const TIn *>(a.beta);
    L.bh_cur = L.cur.b * a.H + sc.hord[L.cur.h];
    L.beta_cur = to_f32(beta_g[L.bh_cur]);
    L.ok = mbar_wait_bounded(&sc.full[0], 0u);
    {
        const StageMeta m0 = sc.meta[0];
        const float al0 = (GATE == STEPQ_GATE_GDN) ? to_f32(alpha_g[L.bh_cur]) : 1.0f;
        if (m0.valid && tid >= DK) row_table<GATE, TIn, ROWS>(stages, a, m0.bits, m0.head, al0, sc, tid);
    }
    __syncthreads();

    int i = 0;
    // the class of heads with per-key-row widths is compiled only into the kernels of pools
    // that have such heads
    bool done = L.template run<4>(i, end4) && L.template run<6>(i, end6);
    if constexpr (ROWS)
        done = done && L.template run<8>(i, end8) && L.template run<0>(i, count);
    else
        done = done && L.template run<8>(i, count);
    const int lane = tid & 31;
    if (lane == 0) bulk_wait_all();
    if (tid == 0 && !done) {
        atomicOr(a.flag, STEPQ_FLAG_TIMEOUT);
        // let the loads still in flight land before the CTA leaves (bounded waits)
        const int issued = i + 2 < count ? i + 3 : count;
        for (int j = i; j < issued; ++j)
            (void)mbar_wait_bounded(&sc.full[j % kStages], uint32_t(j / kStages) & 1u);
    }
}

// ------------------------------------------------------------------------------------------
// FP16 pivot heads (STEPQuant summary, "Method" para 2: the highest-risk units are kept in
// FP16).  The state is binary16, row-major; the step fades, writes and reads out as for the
// quantized heads and stores the updated state rounded to binary16 (nearest, ties to even),
// with no fit.  One CTA of 256 threads per (request, pivot head): warp w owns the 16-column
// panel w, lane l rows l + 32 m, the same column dot products as the quantized kernel with
// rho_i = alpha_i and no column factor.
// ------------------------------------------------------------------------------------------
template <int GATE, typename TIn>
__global__ void __launch_bounds__(kThreads) pivot_kernel(const DecodeArgs a, int npiv)
{
    __shared__ float4 wlo[DK], whi[DK], wrk[DK];
    __shared__ float xd[DV];
    __shared__ float kqw[4];
    const int tid = threadIdx.x;
    const long long item = blockIdx.x;
    const int b = int(item / npiv);
    const int h = a.head_order[a.Hq + int(item % npiv)];
    const int slot = a.slot_ids[b];
    if (slot < 0 || slot >= a.num_slots) {
        if (tid == 0) atomicOr(a.flag, STEPQ_FLAG_BAD_SLOT);
        return;
    }
    const int g = h / a.group;
    const long long bh = (long long)b * a.H + h;
    const long long kqrow = (long long)b * a.Hk + g;
    uint16_t *blk = reinterpret_cast<uint16_t *>(a.pool + (long long)slot * a.slot_stride + a.head_off[h]);
    const TIn *qg = static_cast<const TIn *>(a.q) + kqrow * DK;
    const TIn *kg = static_cast<const TIn *>(a.k) + kqrow * DK;
    const TIn *vg = static_cast<const TIn *>(a.v) + bh * DV;
    const TIn *ag = static_cast<const TIn *>(a.alpha);
    const float beta = to_f32(static_cast<const TIn *>(a.beta)[bh]);

    // row tables (threads 0..127, row tid) and k.q
    if (tid < DK) {
        const float al = to_f32(GATE == STEPQ_GATE_KDA ? ag[bh * DK + tid] : ag[bh]);
        const float k = to_f32(kg[tid]), q = to_f32(qg[tid]);
        const float rk = al * k, rq = al * q;
        wlo[tid] = make_float4(rk, rk, rq, rq);
        whi[tid] = make_float4(rq, rq, rk, rk);
        wrk[tid] = make_float4(al, al, k, k);
        float kq = k * q;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) kq += __shfl_xor_sync(kFull, kq, o);
        if ((tid & 31) == 0) kqw[tid >> 5] = kq;
    }
    const TileIdx<4> ix(tid);
    const int lane = ix.lane, panel = ix.panel;
    const bool upper = (lane & 16) != 0;
    const int col = lane & 15;
    float T[4][PANEL];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint4 *src = reinterpret_cast<const uint4 *>(blk + ix.row(m) * DV + panel * PANEL);
        const uint4 lo = src[0], hi = src[1];
        const uint32_t wv[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&wv[e]));
            T[m][2 * e] = f.x;
            T[m][2 * e + 1] = f.y;
        }
    }
    __syncthreads();
    const float kq = (kqw[0] + kqw[1]) + (kqw[2] + kqw[3]);

    // u_j (lanes 0..15) and y'_j (lanes 16..31) of the panel's columns
    const float4 *wt = upper ? whi : wlo;
    float4 w[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) w[m] = wt[ix.row(m)];
    float A[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 2) {
        float2 s1 = fmul2(make_float2(T[0][j], T[0][j + 1]), make_float2(w[0].x, w[0].y));
        float2 s2 = fmul2(make_float2(T[0][j], T[0][j + 1]), make_float2(w[0].z, w[0].w));
#pragma unroll
        for (int m = 1; m < 4; ++m) {
            s1 = ffma2(make_float2(T[m][j], T[m][j + 1]), make_float2(w[m].x, w[m].y), s1);
            s2 = ffma2(make_float2(T[m][j], T[m][j + 1]), make_float2(w[m].z, w[m].w), s2);
        }
        A[j] = s1.x + __shfl_xor_sync(kFull, s2.x, 16);
        A[j + 1] = s1.y + __shfl_xor_sync(kFull, s2.y, 16);
    }
    reduce_scatter<PANEL, 4, 8, false>(A, lane);
    const float delta = beta * (to_f32(vg[panel * PANEL + col]) - A[0]);
    const float dpair = __shfl_xor_sync(kFull, delta, 16);
    st_global_if(upper, a.y + bh * DV + panel * PANEL + col, fmaf(dpair, kq, A[0]));
    st_shared_if(!upper, xd + panel * PANEL + col, delta);
    __syncwarp();
    float dd[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 t4 = *reinterpret_cast<const float4 *>(xd + panel * PANEL + j);
        dd[j] = t4.x; dd[j + 1] = t4.y; dd[j + 2] = t4.z; dd[j + 3] = t4.w;
    }
    // S_ij = alpha_i S_ij + k_i d_j, stored as binary16 in place
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float4 rk = wrk[ix.row(m)];
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            float2 t2 = fmul2(make_float2(T[m][j], T[m][j + 1]), make_float2(rk.x, rk.y));
            t2 = ffma2(make_float2(rk.z, rk.w), make_float2(dd[j], dd[j + 1]), t2);
            const __half2 hv = __float22half2_rn(t2);
            o[j / 2] = *reinterpret_cast<const uint32_t *>(&hv);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(blk + ix.row(m) * DV + panel * PANEL);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

size_t decode_smem_bytes(int stage_bytes)
{
    return size_t(kStages) * stage_bytes + sizeof(Scratch);
}

// Largest dynamic shared memory any pool can ask for: 8-bit blocks plus four input vectors.
// Every instantiation is opened up to it once, so pools of different shapes can share it.
size_t decode_smem_max()
{
    return decode_smem_bytes((block_bytes(8) + 4 * kIoBytes + 127) / 128 * 128);
}

template <int GATE, typename TIn>
cudaError_t configure_one(stepq_pool *p)
{
    const void *kernels[4] = {reinterpret_cast<const void *>(decode_kernel<GATE, TIn, false, false>),
                              reinterpret_cast<const void *>(decode_kernel<GATE, TIn, true, false>),
                              reinterpret_cast<const void *>(decode_kernel<GATE, TIn, false, true>),
                              reinterpret_cast<const void *>(decode_kernel<GATE, TIn, true, true>)};
    int per_sm_min = 1 << 30;
    for (const void *kern : kernels) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(decode_smem_max()));
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, p->decode_smem);
        if (e != cudaSuccess) return e;
        if (per_sm < per_sm_min) per_sm_min = per_sm;
    }
    if (per_sm_min < 1) return cudaErrorInvalidConfiguration;
    p->decode_grid = per_sm_min * p->num_sms;
    return cudaSuccess;
}

cudaError_t upload_tables()
{
    float h[3][PANEL];
    const int widths[3] = {4, 6, 8};
    for (int b = 0; b < 3; ++b)
        for (int p = 0; p < PANEL; ++p) h[b][p] = 1.0f / pos_scale(widths[b], p);
    return cudaMemcpyToSymbol(kInvPos, h, sizeof(h));
}

// The decode kernel is launched as a programmatic dependent of the previous kernel in the
// stream: its CTAs may start (shared-memory setup, head tables) while that kernel's last
// CTAs finish, and wait for it before touching states, inputs or y.
template <int GATE, typename TIn, bool IMPACT, bool ROWS>
cudaError_t launch_dependent(int grid, size_t smem, cudaStream_t stream, const DecodeArgs &a)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<GATE, TIn, IMPACT, ROWS>, a);
}

template <int GATE, typename TIn>
cudaError_t launch_variant(bool impact, bool rows, int grid, size_t smem, cudaStream_t stream, const DecodeArgs &a)
{
    if (impact)
        return rows ? launch_dependent<GATE, TIn, true, true>(grid, smem, stream, a)
                    : launch_dependent<GATE, TIn, true, false>(grid, smem, stream, a);
    return rows ? launch_dependent<GATE, TIn, false, true>(grid, smem, stream, a)
                : launch_dependent<GATE, TIn, false, false>(grid, smem, stream, a);
}

void count_widths(const uint8_t *bits, int H, DecodeArgs &a)
{
    a.nh4 = a.nh6 = a.nh8 = 0;
    for (int h = 0; h < H; ++h) {
        a.nh4 += bits[h] == 4;
        a.nh6 += bits[h] == 6;
        a.nh8 += bits[h] == 8;
    }
}

}  // namespace

cudaError_t decode_configure(stepq_pool *p)
{
    cudaError_t e = upload_tables();
    if (e != cudaSuccess) return e;
    p->blk_cap = kBlkCap;
    p->stage_bytes = p->gate_mode == STEPQ_GATE_KDA ? stage_bytes_of<STEPQ_GATE_KDA>() : stage_bytes_of<STEPQ_GATE_GDN>();
    p->decode_smem = decode_smem_bytes(p->stage_bytes);
    if (p->gate_mode == STEPQ_GATE_GDN)
        return p->in_dtype == STEPQ_DTYPE_BF16 ? configure_one<STEPQ_GATE_GDN, uint16_t>(p)
                                              : configure_one<STEPQ_GATE_GDN, float>(p);
    return p->in_dtype == STEPQ_DTYPE_BF16 ? configure_one<STEPQ_GATE_KDA, uint16_t>(p)
                                          : configure_one<STEPQ_GATE_KDA, float>(p);
}

cudaError_t launch_decode(const stepq_pool *p, const int32_t *slot_ids, int n, const void *q, const void *k,
                          const void *v, const void *alpha, const void *beta, float *y, cudaStream_t stream)
{
    DecodeArgs a;
    a.pool = p->d_pool;
    a.slot_stride = p->slot_stride;
    a.head_off = p->d_offs;
    a.head_bits = p->d_bits;
    a.head_order = p->d_order;
    a.num_slots = p->num_slots;
    a.H = p->H;
    a.Hk = p->Hk;
    a.group = p->H / p->Hk;
    count_widths(p->bits.data(), p->H, a);
    a.slot_ids = slot_ids;
    a.n = n;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta;
    a.y = y;
    a.flag = p->d_flag;
    a.Hq = p->H - p->npiv;
    a.impact = p->d_impact;
    a.head_blk = p->d_blk;
    a.row_n8 = p->d_rn8;
    a.row_n4 = p->d_rn4;
    a.row_pb = p->d_rpb;
    a.row_perm = p->d_perm;
    // items are dealt round-robin in head-major order, so the CTAs resident at any moment
    // work on one or two heads (one bit width: one code path in the instruction caches)
    // FP16 pivot heads run on their own stream, forked here from the caller's stream: their
    // kernel touches neither the quantized heads nor their rows of y, so it can take the SM
    // slots that free up while the persistent decode grid finishes
    const bool piv = p->npiv > 0;
    if (piv) {
        const cudaError_t e = cudaEventRecord(p->ev_pfork, stream);
        if (e != cudaSuccess) return e;
    }
    const long long total = (long long)n * a.Hq;
    if (total > 0) {
        const int grid = int(total < p->decode_grid ? total : p->decode_grid);
        a.step_b = grid % n;
        a.step_h = grid / n;
        const size_t sm = p->decode_smem;
        const bool rows = p->d_perm != nullptr;
        const bool imp = a.impact != nullptr;
        cudaError_t e;
        if (p->gate_mode == STEPQ_GATE_GDN)
            e = p->in_dtype == STEPQ_DTYPE_BF16 ? launch_variant<STEPQ_GATE_GDN, uint16_t>(imp, rows, grid, sm, stream, a)
                                                : launch_variant<STEPQ_GATE_GDN, float>(imp, rows, grid, sm, stream, a);
        else
            e = p->in_dtype == STEPQ_DTYPE_BF16 ? launch_variant<STEPQ_GATE_KDA, uint16_t>(imp, rows, grid, sm, stream, a)
                                                : launch_variant<STEPQ_GATE_KDA, float>(imp, rows, grid, sm, stream, a);
        if (e != cudaSuccess) return e;
    }
    if (piv) {
        cudaStream_t ps = p->s_piv;
        cudaError_t e = cudaStreamWaitEvent(ps, p->ev_pfork, 0);
        if (e != cudaSuccess) return e;
        const unsigned pgrid = unsigned(n) * unsigned(p->npiv);
        if (p->gate_mode == STEPQ_GATE_GDN) {
            if (p->in_dtype == STEPQ_DTYPE_BF16)
                pivot_kernel<STEPQ_GATE_GDN, uint16_t><<<pgrid, kThreads, 0, ps>>>(a, p->npiv);
            else
                pivot_kernel<STEPQ_GATE_GDN, float><<<pgrid, kThreads, 0, ps>>>(a, p->npiv);
        } else {
            if (p->in_dtype == STEPQ_DTYPE_BF16)
                pivot_kernel<STEPQ_GATE_KDA, uint16_t><<<pgrid, kThreads, 0, ps>>>(a, p->npiv);
            else
                pivot_kernel<STEPQ_GATE_KDA, float><<<pgrid, kThreads, 0, ps>>>(a, p->npiv);
        }
        e = cudaGetLastError();
        // join: everything after this step on the caller's stream sees the pivot heads done
        if (e == cudaSuccess) e = cudaEventRecord(p->ev_pjoin, ps);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, p->ev_pjoin, 0);
        return e;
    }
    return cudaGetLastError();
}

}  // namespace stepq

// ------------------------------------------------------------------------------------------
// stepq_decode_step_noalloc: the same decode kernel for callers that cannot allocate device
// memory.  The caller brings the packed state buffer; the kernel's scratch (the sticky flag
// word and the per-head tables that a pool keeps in its own allocations) lives in a
// file-scope device array instead.
// ------------------------------------------------------------------------------------------
#include <mutex>

namespace stepq {
namespace {

constexpr int kNoallocFlagOffset = 0;                                     // int32 flag word
constexpr int kNoallocOffOffset = 256;                                    // int64[kMaxHeads]
constexpr int kNoallocOrderOffset = kNoallocOffOffset + 8 * kMaxHeads;   // int32[kMaxHeads]
constexpr int kNoallocBitsOffset = kNoallocOrderOffset + 4 * kMaxHeads;  // uint8[kMaxHeads]
constexpr int kNoallocScratchBytes = kNoallocBitsOffset + kMaxHeads;      // 3584 bytes
static_assert(kNoallocScratchBytes == 3584, "scratch size is documented in stepq.h");

// Scratch of the allocation-free entry point.  Every GPU that loads the library holds it
// until the process exits; host code reaches it only through the address returned by
// cudaGetSymbolAddress (the symbol itself is a host-side stand-in).
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

// The scratch contents of one call (flag word cleared, head tables), passed by value as the
// argument of a one-CTA kernel that writes them into the array: no host memory is read by a
// copy, so the call never waits on the host for earlier work of the stream.
struct NoallocImage {
    uint32_t words[kNoallocScratchBytes / 4];
};

__global__ void __launch_bounds__(256) noalloc_fill_kernel(const NoallocImage img)
{
    uint32_t *dst = reinterpret_cast<uint32_t *>(g_noalloc_scratch);
    for (int i = threadIdx.x; i < kNoallocScratchBytes / 4; i += blockDim.x) dst[i] = img.words[i];
}

struct NoallocDevice {
    bool ready = false;
    uint8_t *scratch = nullptr;         // device address of g_noalloc_scratch on this device
    int num_sms = 0;
};
constexpr int kNoallocMaxDevices = 64;
NoallocDevice g_noalloc_dev[kNoallocMaxDevices];
std::mutex g_noalloc_mu;

// Once per device, with that device current: resolve the scratch address and open the
// kernel instantiations up to their largest shared-memory size.
cudaError_t noalloc_setup(int dev, NoallocDevice **out)
{
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocDevice &d = g_noalloc_dev[dev];
    if (!d.ready) {
        void *ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = upload_tables();
        if (e != cudaSuccess) return e;
        const int smem = int(decode_smem_max());
        e = cudaFuncSetAttribute(decode_kernel<STEPQ_GATE_GDN, float, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_kernel<STEPQ_GATE_GDN, uint16_t, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_kernel<STEPQ_GATE_KDA, float, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_kernel<STEPQ_GATE_KDA, uint16_t, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        d.scratch = static_cast<uint8_t *>(ptr);
        d.ready = true;
    }
    *out = &d;
    return cudaSuccess;
}

template <int GATE, typename TIn>
cudaError_t noalloc_launch(const DecodeArgs &a0, int num_sms, size_t smem, cudaStream_t stream)
{
    DecodeArgs a = a0;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<GATE, TIn, false, false>, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long total = (long long)a.n * a.H;
    const long long cap = (long long)per_sm * num_sms;
    const int grid = int(total < cap ? total : cap);
    a.step_b = grid % a.n;
    a.step_h = grid / a.n;
    decode_kernel<GATE, TIn, false, false><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace
}  // namespace stepq

extern "C" int stepq_decode_step_noalloc(const stepq_pool_desc *desc, uint8_t *state, const int32_t *slot_ids,
                                         int32_t n, const void *q, const void *k, const void *v, const void *alpha,
                                         const void *beta, float *y, int32_t *flag_out, stepq_stream stream)
{
    using namespace stepq;
    const NvtxRange range("stepq_decode_step_noalloc");
    if (!desc || !desc->head_bits || n < 0) return STEPQ_INVALID_ARG;
    if (desc->num_slots <= 0 || desc->num_heads <= 0 || desc->num_key_heads <= 0) return STEPQ_INVALID_ARG;
    if (desc->num_heads % desc->num_key_heads != 0) return STEPQ_INVALID_ARG;
    if (desc->num_heads > kMaxHeads) return STEPQ_UNSUPPORTED;       // scratch holds kMaxHeads heads
    if (desc->gate_mode != STEPQ_GATE_GDN && desc->gate_mode != STEPQ_GATE_KDA) return STEPQ_INVALID_ARG;
    if (desc->in_dtype != STEPQ_DTYPE_F32 && desc->in_dtype != STEPQ_DTYPE_BF16) return STEPQ_INVALID_ARG;
    if (desc->d_k != DK || desc->d_v != DV) return STEPQ_UNSUPPORTED;
    const int H = desc->num_heads;
    for (int h = 0; h < H; ++h) {
        const int b = desc->head_bits[h];
        if (b != 4 && b != 6 && b != 8) return STEPQ_UNSUPPORTED;
    }
    if (n > desc->num_slots || n > 65535) return STEPQ_INVALID_ARG;
    if (n == 0) return STEPQ_OK;
    auto al = [](const void *p, uintptr_t m) { return (reinterpret_cast<uintptr_t>(p) & (m - 1)) == 0; };
    const size_t esz = desc->in_dtype == STEPQ_DTYPE_BF16 ? 2 : 4;
    if (!state || !slot_ids || !q || !k || !v || !alpha || !beta || !y) return STEPQ_INVALID_ARG;
    if (!al(state, 128) || !al(slot_ids, 4) || !al(q, 16) || !al(k, 16) || !al(v, 16) || !al(y, 4) ||
        !al(beta, esz) || !(desc->gate_mode == STEPQ_GATE_KDA ? al(alpha, 16) : al(alpha, esz)) ||
        (flag_out && !al(flag_out, 4)))
        return STEPQ_INVALID_ARG;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return STEPQ_CUDA_ERROR;
    NoallocDevice *nd = nullptr;
    if (noalloc_setup(dev, &nd) != cudaSuccess) return STEPQ_CUDA_ERROR;

    // head tables (and a cleared flag word) as one image of the scratch, written by a kernel
    NoallocImage img = {};
    uint8_t *image = reinterpret_cast<uint8_t *>(img.words);
    long long *off = reinterpret_cast<long long *>(image + kNoallocOffOffset);
    int32_t *order = reinterpret_cast<int32_t *>(image + kNoallocOrderOffset);
    uint8_t *bits = image + kNoallocBitsOffset;
    long long stride = 0;
    int nord = 0;
    for (int h = 0; h < H; ++h) {
        off[h] = stride;
        bits[h] = desc->head_bits[h];
        stride += block_bytes(bits[h]);
    }
    for (int w = 4; w <= 8; w += 2)
        for (int h = 0; h < H; ++h)
            if (bits[h] == w) order[nord++] = h;
    noalloc_fill_kernel<<<1, 256, 0, stream>>>(img);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return STEPQ_CUDA_ERROR;

    DecodeArgs a;
    a.pool = state;
    a.slot_stride = stride;
    a.head_off = reinterpret_cast<const long long *>(nd->scratch + kNoallocOffOffset);
    a.head_bits = nd->scratch + kNoallocBitsOffset;
    a.head_order = reinterpret_cast<const int32_t *>(nd->scratch + kNoallocOrderOffset);
    a.num_slots = desc->num_slots;
    a.H = H;
    a.Hk = desc->num_key_heads;
    a.group = H / desc->num_key_heads;
    a.Hq = H;
    a.impact = nullptr;
    a.head_blk = nullptr;                   // every head here has a uniform width
    a.row_n8 = a.row_n4 = a.row_perm = nullptr;
    a.row_pb = nullptr;
    count_widths(bits, H, a);
    a.slot_ids = slot_ids;
    a.n = n;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta;
    a.y = y;
    a.flag = reinterpret_cast<int *>(nd->scratch + kNoallocFlagOffset);
    const size_t smem = decode_smem_bytes(desc->gate_mode == STEPQ_GATE_KDA ? stage_bytes_of<STEPQ_GATE_KDA>()
                                                                        : stage_bytes_of<STEPQ_GATE_GDN>());
    if (desc->gate_mode == STEPQ_GATE_GDN)
        e = desc->in_dtype == STEPQ_DTYPE_BF16 ? noalloc_launch<STEPQ_GATE_GDN, uint16_t>(a, nd->num_sms, smem, stream)
                                               : noalloc_launch<STEPQ_GATE_GDN, float>(a, nd->num_sms, smem, stream);
    else
        e = desc->in_dtype == STEPQ_DTYPE_BF16 ? noalloc_launch<STEPQ_GATE_KDA, uint16_t>(a, nd->num_sms, smem, stream)
                                               : noalloc_launch<STEPQ_GATE_KDA, float>(a, nd->num_sms, smem, stream);
    if (e != cudaSuccess) return STEPQ_CUDA_ERROR;
    if (flag_out) {
        e = cudaMemcpyAsync(flag_out, nd->scratch + kNoallocFlagOffset, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                            stream);
        if (e != cudaSuccess) return STEPQ_CUDA_ERROR;
    }
    return STEPQ_OK;
}
