// stepq_kernels.cu -- sm_100a kernels of the quantized gated Delta-rule decode step.
//
// decode_kernel: one fused pass per (request, value head) state, persistent CTAs.
//   HBM -> shared: 1-D bulk async copies (packed head block, q, k, v, per-channel
//   gate) into a 4-stage ring, completion on mbarriers (bounded waits).
//   shared -> registers: each thread unpacks ROWS rows x 16 columns of codes.
//   In registers: dequantize + fade, the two column dot products S'^T k and S'^T q,
//   the Delta write, the readout, the clip-free column/row fit, round-half-even
//   quantization and repacking.  The packed block is written back over its stage
//   buffer and stored with one bulk copy, so each state is read once and written
//   once.  (STEPQuant summary, "Method": update the reconstructed state in floating
//   point, compute the output, then quantize for storage; "Paper Explained", "The
//   mechanism: rewriting state with the delta rule".)
// load_fp32_kernel / dump_fp32_kernel / copy_slots_kernel: pool I/O.
#include <cfloat>
#include <cstdint>

#include "stepq_internal.h"
#include "stepq_tile.cuh"

namespace stepq {

constexpr int kStages = 4;
constexpr int kIoBytes = 512;       // stage room for one 128-vector input (fp32 or bf16)
constexpr int kRpStride = 12;       // padded row stride of the row-maxima exchange (floats)

struct StageMeta {
    long long dst;                  // byte offset of the head block in the pool
    int valid;
    int bits;
};

struct DecodeArgs {
    uint8_t *pool;
    long long slot_stride;
    const long long *head_off;
    const uint8_t *head_bits;
    int num_slots, H, Hk, group;
    const int32_t *slot_ids;
    int n;
    const void *q, *k, *v, *alpha, *beta;
    float *y;
    int *flag;
    int blk_cap, stage_bytes;
};

// ------------------------------------------------------------------------------------------
// Fit + quantize + pack of a register tile (the updated state S) -- shared by the decode and
// load kernels.  On return S holds garbage.  Writes c (writer lanes), r (panel-0 threads)
// and the packed codes of the thread's rows.  Contains one __syncthreads (row maxima).
// `ok` is folded into that barrier: returns false on every thread if any thread passed false.
// ------------------------------------------------------------------------------------------
template <int ROWS, int BITS>
__device__ __forceinline__ bool fit_quantize_pack(float (&S)[ROWS][PANEL], const TileIdx<ROWS> &ix,
                                                  float *rp, float *xc, uint8_t *codes_out,
                                                  float *r_out, float *c_out, bool ok)
{
    using L = Layout<ROWS>;
    constexpr int QM = qmax_of(BITS);
    constexpr float MAG = kTwo23 + float(1 << (BITS - 1));

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
        rp[ix.row(m) * kRpStride + ix.panel] = a;
    }
    if (__syncthreads_or(!ok)) return false;
    // r_i = max_j (|S_ij| / c_j) / qmax (correctly rounded division); quantize the rows
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        const int row = ix.row(m);
        const float4 a = *reinterpret_cast<const float4 *>(rp + row * kRpStride);
        const float4 b = *reinterpret_cast<const float4 *>(rp + row * kRpStride + 4);
        const float mr = max3(max3(a.x, a.y, a.z), max3(a.w, b.x, b.y), fmaxf(b.z, b.w));
        const float r = mr / float(QM);
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
        pack_seg<BITS>(u, codes_out + ix.panel * panel_bytes(BITS) + row * seg_bytes(BITS));
    }
    return true;
}

// ------------------------------------------------------------------------------------------
// The fused decode step for one state held in a ring stage.  Returns false (on every
// thread) when some thread saw a failed wait.
// ------------------------------------------------------------------------------------------
template <int ROWS, int GATE, typename TIn, int BITS>
__device__ __forceinline__ bool decode_item(uint8_t *stage, const DecodeArgs &a, const TileIdx<ROWS> &ix,
                                            long long it, float alpha_s, float beta, float *rp,
                                            float *xd, float *xc, bool ok)
{
    using L = Layout<ROWS>;
    uint8_t *codes = stage;
    float *r_io = reinterpret_cast<float *>(stage + codes_bytes(BITS));
    float *c_io = r_io + DK;
    const TIn *qs = reinterpret_cast<const TIn *>(stage + a.blk_cap);
    const TIn *ks = reinterpret_cast<const TIn *>(stage + a.blk_cap + kIoBytes);
    const TIn *vs = reinterpret_cast<const TIn *>(stage + a.blk_cap + 2 * kIoBytes);
    const TIn *as = reinterpret_cast<const TIn *>(stage + a.blk_cap + 3 * kIoBytes);

    // per-row factors: rho_i = alpha_i r_i (fade folded into the row factor), k_i, q_i
    float rho[ROWS], kq2[ROWS][2];
    float kq = 0.0f;
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        const int row = ix.row(m);
        const float al = (GATE == STEPQ_GATE_KDA) ? to_f32(as[row]) : alpha_s;
        rho[m] = al * r_io[row];
        kq2[m][0] = to_f32(ks[row]);
        kq2[m][1] = to_f32(qs[row]);
        kq = fmaf(kq2[m][0], kq2[m][1], kq);
    }
    // column factors c_j / (position scale of the unpacked field): exact power-of-two scaling
    float cc[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(c_io + ix.panel * PANEL + j);
        cc[j] = t.x * (1.0f / pos_scale(BITS, j));
        cc[j + 1] = t.y * (1.0f / pos_scale(BITS, j + 1));
        cc[j + 2] = t.z * (1.0f / pos_scale(BITS, j + 2));
        cc[j + 3] = t.w * (1.0f / pos_scale(BITS, j + 3));
    }
    // dequantize + fade: S'_ij = Q_ij * (rho_i * c_j)
    float S[ROWS][PANEL];
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        load_codes<BITS>(codes + ix.panel * panel_bytes(BITS) + ix.row(m) * seg_bytes(BITS), S[m]);
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            const float2 sc = fmul2(make_float2(rho[m], rho[m]), make_float2(cc[j], cc[j + 1]));
            const float2 s = fmul2(make_float2(S[m][j], S[m][j + 1]), sc);
            S[m][j] = s.x;
            S[m][j + 1] = s.y;
        }
    }
    // column dot products over the thread's rows: (u_j, y'_j) = sum_i S'_ij (k_i, q_i)
    float acc[2 * PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; ++j) {
        float2 t = fmul2(make_float2(S[0][j], S[0][j]), make_float2(kq2[0][0], kq2[0][1]));
#pragma unroll
        for (int m = 1; m < ROWS; ++m)
            t = ffma2(make_float2(S[m][j], S[m][j]), make_float2(kq2[m][0], kq2[m][1]), t);
        acc[2 * j] = t.x;
        acc[2 * j + 1] = t.y;
    }
    // ... and over the panel's lanes
    reduce_scatter<2 * PANEL, L::LOG_LP, L::LP / 2, false>(acc, ix.lane);
#pragma unroll
    for (int o = L::LP / 2; o >= 1; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);

    // Delta write coefficients delta_j = beta (v_j - u_j) and readout y_j = y'_j + (k.q) delta_j
    float *xdp = xd + ix.panel * PANEL;
    const long long yrow = it * DV + ix.panel * PANEL;
    if (L::LP == 32) {
        const int col = ix.lane >> 1;
        const float delta = beta * (to_f32(vs[ix.panel * PANEL + col]) - acc[0]);
        const float d_pair = __shfl_xor_sync(0xffffffffu, delta, 1);
        if (ix.lane & 1) {
            a.y[yrow + col] = fmaf(d_pair, kq, acc[0]);
        } else {
            xdp[col] = delta;
        }
    } else {
        const int col = ix.rl;
        const float delta = beta * (to_f32(vs[ix.panel * PANEL + col]) - acc[0]);
        a.y[yrow + col] = fmaf(delta, kq, acc[1]);
        xdp[col] = delta;
    }
    __syncwarp();
    float dl[PANEL];
#pragma unroll
    for (int j = 0; j < PANEL; j += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(xdp + j);
        dl[j] = t.x; dl[j + 1] = t.y; dl[j + 2] = t.z; dl[j + 3] = t.w;
    }
    // S_ij = S'_ij + k_i delta_j  (the updated, unquantized state)
#pragma unroll
    for (int m = 0; m < ROWS; ++m)
#pragma unroll
        for (int j = 0; j < PANEL; j += 2) {
            const float2 s = ffma2(make_float2(kq2[m][0], kq2[m][0]), make_float2(dl[j], dl[j + 1]),
                                   make_float2(S[m][j], S[m][j + 1]));
            S[m][j] = s.x;
            S[m][j + 1] = s.y;
        }
    // refit + requantize + repack in place over the stage buffer
    return fit_quantize_pack<ROWS, BITS>(S, ix, rp, xc, codes, r_io, c_io, ok);
}

template <int ROWS, int GATE, typename TIn>
__global__ void __launch_bounds__(Layout<ROWS>::NT, 2) decode_kernel(const DecodeArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *stages = smem;
    float *rp = reinterpret_cast<float *>(smem + kStages * a.stage_bytes);
    float *xd = rp + DK * kRpStride;
    float *xc = xd + NPANEL * PANEL;
    StageMeta *meta = reinterpret_cast<StageMeta *>(xc + NPANEL * PANEL);
    uint64_t *bars = reinterpret_cast<uint64_t *>(meta + kStages);

    const int tid = threadIdx.x;
    const long long total = (long long)a.n * a.H;
    const long long G = gridDim.x;
    const long long first = blockIdx.x;
    if (first >= total) return;
    const int count = int((total - first + G - 1) / G);
    constexpr int esz = sizeof(TIn);

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();

    // ---- producer (thread 0): bulk-copy item j's inputs into stage j % kStages
    int slot_next = 0;          // slot id of the next item to issue (prefetched)
    int issued = 0;
    auto item_index = [&](int j) { return first + (long long)j * G; };
    auto issue = [&](int j) {
        const long long it = item_index(j);
        const int b = int(it / a.H), h = int(it % a.H);
        const int st = j % kStages;
        const int slot = slot_next;
        if (j + 1 < count) slot_next = __ldg(a.slot_ids + item_index(j + 1) / a.H);
        uint8_t *stage = stages + st * a.stage_bytes;
        StageMeta &mt = meta[st];
        if (slot < 0 || slot >= a.num_slots) {
            mt.valid = 0;
            atomicOr(a.flag, STEPQ_FLAG_BAD_SLOT);
            mbar_arrive(&bars[st]);
        } else {
            const int bits = __ldg(a.head_bits + h);
            const uint32_t bb = uint32_t(block_bytes(bits));
            const int g = h / a.group;
            mt.valid = 1;
            mt.bits = bits;
            mt.dst = (long long)slot * a.slot_stride + __ldg(a.head_off + h);
            const uint32_t io = DK * esz;
            const uint32_t tx = bb + 3 * io + (GATE == STEPQ_GATE_KDA ? io : 0u);
            mbar_arrive_expect_tx(&bars[st], tx);
            bulk_g2s(stage, a.pool + mt.dst, bb, &bars[st]);
            const uint8_t *q8 = static_cast<const uint8_t *>(a.q);
            const uint8_t *k8 = static_cast<const uint8_t *>(a.k);
            const uint8_t *v8 = static_cast<const uint8_t *>(a.v);
            bulk_g2s(stage + a.blk_cap, q8 + ((long long)b * a.Hk + g) * io, io, &bars[st]);
            bulk_g2s(stage + a.blk_cap + kIoBytes, k8 + ((long long)b * a.Hk + g) * io, io, &bars[st]);
            bulk_g2s(stage + a.blk_cap + 2 * kIoBytes, v8 + it * io, io, &bars[st]);
            if (GATE == STEPQ_GATE_KDA)
                bulk_g2s(stage + a.blk_cap + 3 * kIoBytes, static_cast<const uint8_t *>(a.alpha) + it * io,
                         io, &bars[st]);
        }
        issued = j + 1;
    };
    if (tid == 0) {
        slot_next = __ldg(a.slot_ids + first / a.H);
        issue(0);
        if (count > 1) issue(1);
    }

    const TileIdx<ROWS> ix(tid);
    const TIn *alpha_g = static_cast<const TIn *>(a.alpha);
    const TIn *beta_g = static_cast<const TIn *>(a.beta);
    // per-item scalar gates, loaded one item ahead by every thread (broadcast loads)
    float beta_cur = to_f32(beta_g[first]);
    float alpha_cur = (GATE == STEPQ_GATE_GDN) ? to_f32(alpha_g[first]) : 1.0f;

    int aborted_at = -1;
    for (int i = 0; i < count; ++i) {
        const int st = i % kStages;
        if (tid == 0 && i + 2 < count) {
            bulk_wait_read<1>();              // the store of item i-2 no longer reads stage (i+2)%4
            issue(i + 2);
        }
        float beta_next = 0.0f, alpha_next = 1.0f;
        if (i + 1 < count) {
            const long long nx = item_index(i + 1);
            beta_next = to_f32(beta_g[nx]);
            if (GATE == STEPQ_GATE_GDN) alpha_next = to_f32(alpha_g[nx]);
        }
        const bool ok = mbar_wait_bounded(&bars[st], uint32_t(i / kStages) & 1u);
        const StageMeta mt = meta[st];
        const long long it = item_index(i);
        uint8_t *stage = stages + st * a.stage_bytes;
        bool alive = true;
        if (!mt.valid) {
            alive = !__syncthreads_or(!ok);
        } else if (mt.bits == 4) {
            alive = decode_item<ROWS, GATE, TIn, 4>(stage, a, ix, it, alpha_cur, beta_cur, rp, xd, xc, ok);
        } else if (mt.bits == 6) {
            alive = decode_item<ROWS, GATE, TIn, 6>(stage, a, ix, it, alpha_cur, beta_cur, rp, xd, xc, ok);
        } else {
            alive = decode_item<ROWS, GATE, TIn, 8>(stage, a, ix, it, alpha_cur, beta_cur, rp, xd, xc, ok);
        }
        if (!alive) {
            aborted_at = i;
            break;
        }
        if (mt.valid) {
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) bulk_s2g(a.pool + mt.dst, stage, uint32_t(block_bytes(mt.bits)));
        }
        if (tid == 0) bulk_commit();
        beta_cur = beta_next;
        alpha_cur = alpha_next;
    }
    if (tid == 0) {
        if (aborted_at >= 0) {
            atomicOr(a.flag, STEPQ_FLAG_TIMEOUT);
            // let the loads still in flight land before the CTA leaves (bounded waits)
            for (int j = aborted_at; j < issued; ++j)
                (void)mbar_wait_bounded(&bars[j % kStages], uint32_t(j / kStages) & 1u);
        }
        bulk_wait_all();
    }
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
};

template <int BITS>
__device__ __forceinline__ void load_fp32_item(const IoArgs &a, uint8_t *blk, const float *S,
                                               const TileIdx<4> &ix, float *rp, float *xc)
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
    fit_quantize_pack<4, BITS>(T, ix, rp, xc, blk, r_out, r_out + DK, true);
}

__global__ void __launch_bounds__(256) load_fp32_kernel(const IoArgs a, const float *S)
{
    __shared__ __align__(16) float rp[DK * kRpStride];
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
    case 4: load_fp32_item<4>(a, blk, Si, ix, rp, xc); break;
    case 6: load_fp32_item<6>(a, blk, Si, ix, rp, xc); break;
    default: load_fp32_item<8>(a, blk, Si, ix, rp, xc); break;
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
    case 4: dump_fp32_item<4>(blk, Si, ix); break;
    case 6: dump_fp32_item<6>(blk, Si, ix); break;
    default: dump_fp32_item<8>(blk, Si, ix); break;
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
// Launchers
// ------------------------------------------------------------------------------------------
namespace {

constexpr int kDecodeRows = 4;

size_t decode_smem_bytes(int stage_bytes)
{
    return size_t(kStages) * stage_bytes + sizeof(float) * (DK * kRpStride + 2 * NPANEL * PANEL) +
           sizeof(StageMeta) * kStages + sizeof(uint64_t) * kStages;
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
    auto kern = decode_kernel<kDecodeRows, GATE, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(decode_smem_max()));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Layout<kDecodeRows>::NT, p->decode_smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    p->decode_grid = per_sm * p->num_sms;
    return cudaSuccess;
}

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
    return a;
}

}  // namespace

cudaError_t decode_configure(stepq_pool *p)
{
    p->blk_cap = p->max_block;
    const int io = (p->gate_mode == STEPQ_GATE_KDA ? 4 : 3) * kIoBytes;
    p->stage_bytes = (p->blk_cap + io + 127) / 128 * 128;
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
    a.num_slots = p->num_slots;
    a.H = p->H;
    a.Hk = p->Hk;
    a.group = p->H / p->Hk;
    a.slot_ids = slot_ids;
    a.n = n;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta;
    a.y = y;
    a.flag = p->d_flag;
    a.blk_cap = p->blk_cap;
    a.stage_bytes = p->stage_bytes;
    const long long total = (long long)n * p->H;
    const int grid = int(total < p->decode_grid ? total : p->decode_grid);
    const dim3 block(Layout<kDecodeRows>::NT);
    if (p->gate_mode == STEPQ_GATE_GDN) {
        if (p->in_dtype == STEPQ_DTYPE_BF16)
            decode_kernel<kDecodeRows, STEPQ_GATE_GDN, uint16_t><<<grid, block, p->decode_smem, stream>>>(a);
        else
            decode_kernel<kDecodeRows, STEPQ_GATE_GDN, float><<<grid, block, p->decode_smem, stream>>>(a);
    } else {
        if (p->in_dtype == STEPQ_DTYPE_BF16)
            decode_kernel<kDecodeRows, STEPQ_GATE_KDA, uint16_t><<<grid, block, p->decode_smem, stream>>>(a);
        else
            decode_kernel<kDecodeRows, STEPQ_GATE_KDA, float><<<grid, block, p->decode_smem, stream>>>(a);
    }
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
