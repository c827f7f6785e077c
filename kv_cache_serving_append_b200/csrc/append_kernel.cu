// append_kernel.cu -- fused cache append: 3D axial RoPE (Q, K), per-(token,
// head) amax, scale amax/448 and E4M3 cast, in one pass over bf16 Q/K/V.
//
// Source of the operation: aidose.in, "Runway explains how it serves a 57B
// video model in real time", third paragraph (RoPE and FP8 quantisation done
// once, as a frame enters the cache); pttl.gr, section "Από οκτώ H100 σε
// τέσσερις" (the transformation happens at write time).  The exact arithmetic
// (fixed fp32 rounding order, RNE saturating E4M3, reciprocal multiply) is the
// library's definition, restated in rtv.h.
//
// Work split: blockIdx.y picks Q, K or V; a half-warp (16 lanes) owns one
// token row at a time (grid-stride over the chunk's rows) and walks that
// row's heads, keeping kItems loads in flight (the load of head h + kItems is
// issued as soon as head h is done).  For V, lane i loads the D/16 contiguous
// elements [D/16*i, D/16*(i+1)) of a (row, head) item (16 bytes at D = 128),
// so the item is read in full sectors.  For Q and K, lane i holds D/32
// rotation pairs (j, j + n/2) of one RoPE segment, both members loaded by
// itself: the rotation needs no shuffle, and the lane's D/32 cos/sin pairs,
// which depend only on the row, stay in registers for all of the row's heads.
// The arithmetic keeps the library's rounding order bit for bit while issuing
// two elements per instruction where that is exact: the RoPE products and sum
// as f32x2 FMAs whose -0 addend and unit factor are kernel parameters (nothing
// the compiler could fold into a fused multiply-add), the quantising products
// as f32x2 multiplies, and the scale amax/448 as a product with the
// reciprocal corrected by its FMA residual.  Every input byte is read once and
// every code byte written once.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "rtv_internal.h"

namespace rtv {
namespace {

constexpr int kThreads = 256;
constexpr int kGroups = kThreads / 16;   // half-warps (rows in flight) per block
constexpr int kItems = 3;                // loads in flight per half-warp

template <int E>
struct Vec;
template <>
struct Vec<8> { using T = uint4; };
template <>
struct Vec<4> { using T = uint2; };
template <>
struct Vec<2> { using T = uint32_t; };

__device__ __forceinline__ void unpack_bf16(const uint4& v, float* x)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack_bf16(const uint2& v, float* x)
{
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xffff0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xffff0000u);
}
__device__ __forceinline__ void unpack_bf16(const uint32_t& v, float* x)
{
    x[0] = __uint_as_float(v << 16);
    x[1] = __uint_as_float(v & 0xffff0000u);
}

__device__ __forceinline__ uint64_t pack2(float a, float b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
// Two IEEE round-to-nearest products in one instruction (bit-identical to
// two __fmul_rn; the products feed only the E4M3 conversion).
__device__ __forceinline__ float2 mul2(float a, float b, float c)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pack2(a, b)), "l"(pack2(c, c)));
    float2 o;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(r));
    return o;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t r, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}

// Items with amax below this are stored as zero (zero codes, scale 0): the
// fp32 reciprocal 448/amax would overflow there and turn zeros into NaN.
constexpr float kMinAmax = 0x1p-119f;

// amax / 448 for amax >= kMinAmax, correctly rounded: the product with
// RN(1/448) corrected once by its FMA residual (Markstein's correction step),
// which equals IEEE division for every positive finite float from 2^-120 up.
__device__ __forceinline__ float div448(float a)
{
    constexpr float z = 1.0f / 448.0f;
    const float q0 = __fmul_rn(a, z);
    const float r = __fmaf_rn(-q0, 448.f, a);
    return __fmaf_rn(r, z, q0);
}

// E4M3 round-to-nearest-even with saturation to +-448 (hardware cvt).
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi)
{
    return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

template <int E>
__device__ __forceinline__ void store_codes(uint8_t* dst, const float* y, float inv);
__device__ __forceinline__ uint16_t e4m3x2(float2 v) { return e4m3x2(v.x, v.y); }
template <>
__device__ __forceinline__ void store_codes<8>(uint8_t* dst, const float* y, float inv)
{
    uint32_t w0 = e4m3x2(mul2(y[0], y[1], inv)) | ((uint32_t)e4m3x2(mul2(y[2], y[3], inv)) << 16);
    uint32_t w1 = e4m3x2(mul2(y[4], y[5], inv)) | ((uint32_t)e4m3x2(mul2(y[6], y[7], inv)) << 16);
    *reinterpret_cast<uint2*>(dst) = make_uint2(w0, w1);
}
template <>
__device__ __forceinline__ void store_codes<4>(uint8_t* dst, const float* y, float inv)
{
    uint32_t w0 = e4m3x2(mul2(y[0], y[1], inv)) | ((uint32_t)e4m3x2(mul2(y[2], y[3], inv)) << 16);
    *reinterpret_cast<uint32_t*>(dst) = w0;
}

// V: lane i of a half-warp holds the E = D/16 contiguous elements
// [E*i, E*i + E) of a (row, head) item -- 16 bytes at D = 128 -- so the 16
// lanes read the item in full 32-byte sectors.  The largest scale of every
// (frame, head) is kept in shared memory for the attention's Sv.
template <int D>
__device__ __forceinline__ void append_rows_v(const AppendParams& p, unsigned int (*s_vmax)[kMaxHeads])
{
    constexpr int E = D / 16;
    using V = typename Vec<E>::T;
    constexpr int tensor = 2;
    const int H = p.H, T = p.T;
    const int n_rows = p.n_frames * T;
    const int lane16 = threadIdx.x & 15;
    const uint16_t* src = p.src[tensor];
    // Rows are visited grid-stride; the trip count is the same for the two
    // half-warps of a warp only if both have a row, so the loop runs while
    // either has one (full-warp shuffles need all 32 lanes) and the other
    // idles through it without memory access.
    const int stride = gridDim.x * kGroups;
    const int row_pair0 = blockIdx.x * kGroups + ((threadIdx.x >> 4) & ~1);
    for (int rbase = row_pair0; rbase < n_rows; rbase += stride) {
        const int row = rbase + ((threadIdx.x >> 4) & 1);
        const bool row_ok = row < n_rows;
        const int frame = row_ok ? row / T : 0;
        const int tok = row_ok ? row - frame * T : 0;

        const V* item = reinterpret_cast<const V*>(src + (size_t)row * H * D + lane16 * E);
        V raw[kItems];
#pragma unroll
        for (int u = 0; u < kItems; ++u) raw[u] = (row_ok && u < H) ? __ldcs(item + (size_t)u * (D / E)) : V{};

        // destination of head 0 of this row, and the step from one head to the next
        const int slot = p.ring ? p.ring->staged_slot[frame] : p.slot[frame];
        uint8_t* dst = p.kv_codes[tensor - 1] + ((size_t)slot * H * T + tok) * D + lane16 * E;
        float* sdst = p.kv_scales[tensor - 1] + (size_t)slot * H * p.scale_pitch + tok;
        const size_t dst_step = (size_t)T * D, sdst_step = p.scale_pitch;

        for (int h0 = 0; h0 < H; h0 += kItems) {
#pragma unroll
            for (int u = 0; u < kItems; ++u) {
                const int h = h0 + u;
                const V cur = raw[u];
                // keep kItems loads in flight: the next load of this register
                if (row_ok && h + kItems < H) raw[u] = __ldcs(item + (size_t)(h + kItems) * (D / E));
                float y[E];
                unpack_bf16(cur, y);
                float amax = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[e]));
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (!row_ok || h >= H) continue;
                const bool keep = amax >= kMinAmax;
                const float inv = keep ? __fdiv_rn(448.f, amax) : 0.f;
                store_codes<E>(dst + (size_t)h * dst_step, y, inv);
                if (lane16 == 0) {
                    const float scale = keep ? div448(amax) : 0.f;
                    sdst[(size_t)h * sdst_step] = scale;
                    atomicMax(&s_vmax[frame][h], __float_as_uint(scale));
                }
            }
        }
    }
}

// Q and K.  Lane i of a half-warp holds E/2 rotation pairs (j, j + n/2) of one
// RoPE segment -- the pairs E/2*i .. E/2*i + E/2 - 1 in segment order (frame,
// grid row, grid column) -- so both members of every pair are its own: two
// E/2-element loads per (row, head) item, no shuffle, and one cos/sin pair per
// rotation pair for the whole row, held in registers.
//   x'[j]       = fl(fl(x[j] c) + fl(x[j+n/2] (-s)))   (= x[j] c - x[j+n/2] s)
//   x'[j + n/2] = fl(fl(x[j+n/2] c) + fl(x[j] s))
// two elements per f32x2 FMA (the -0 addend and unit factor are parameters).
template <int D>
__device__ __forceinline__ void append_rows_rope(const AppendParams& p, int tensor)
{
    constexpr int E = D / 16;
    constexpr int P = E / 2;                 // rotation pairs per lane
    using HV = typename Vec<P>::T;
    const int H = p.H, T = p.T;
    const int n_rows = p.n_frames * T;
    const int pt = p.n_t / 2, ph = p.n_h / 2, pw = p.n_w / 2;
    const int lane16 = threadIdx.x & 15;

    const int pq = lane16 * P;               // first pair (global pair order) of this lane
    int seg = 0, half = pt, r0 = pq, seg_lo = 0;
    if (pq >= pt + ph) {
        seg = 2; half = pw; r0 = pq - pt - ph; seg_lo = p.n_t + p.n_h;
    } else if (pq >= pt) {
        seg = 1; half = ph; r0 = pq - pt; seg_lo = p.n_t;
    }
    const int ea = seg_lo + r0, eb = ea + half;   // element offsets of the two runs
    const uint64_t mz2 = pack2(p.neg_zero, p.neg_zero), one2 = pack2(p.one, p.one);

    const uint16_t* src = p.src[tensor];
    const int stride = gridDim.x * kGroups;
    const int row_pair0 = blockIdx.x * kGroups + ((threadIdx.x >> 4) & ~1);
    for (int rbase = row_pair0; rbase < n_rows; rbase += stride) {
        const int row = rbase + ((threadIdx.x >> 4) & 1);
        const bool row_ok = row < n_rows;
        const int frame = row_ok ? row / T : 0;
        const int tok = row_ok ? row - frame * T : 0;

        float cc[P], ss[P];
        if (seg == 0) {
            const float (*tt)[kMaxRopeHalf] = p.ring ? p.ring->t_table[frame] : p.t_table[frame];
#pragma unroll
            for (int k = 0; k < P; ++k) {
                cc[k] = tt[0][r0 + k];
                ss[k] = tt[1][r0 + k];
            }
        } else {
            const float* t = seg == 1 ? p.h_table + (size_t)(tok / p.grid_w) * 2 * ph
                                      : p.w_table + (size_t)(tok % p.grid_w) * 2 * pw;
#pragma unroll
            for (int k = 0; k < P; ++k) {
                cc[k] = __ldg(t + r0 + k);
                ss[k] = __ldg(t + half + r0 + k);
            }
        }

        const uint16_t* item = src + (size_t)row * H * D;
        HV ra[kItems], rb[kItems];
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
            ra[u] = (row_ok && u < H) ? __ldcs(reinterpret_cast<const HV*>(item + u * D + ea)) : HV{};
            rb[u] = (row_ok && u < H) ? __ldcs(reinterpret_cast<const HV*>(item + u * D + eb)) : HV{};
        }

        uint8_t* dst;
        float* sdst;
        size_t dst_step, sdst_step;
        if (tensor == 0) {
            dst = p.q_codes + (size_t)row * D;
            sdst = p.q_scales + row;
            dst_step = (size_t)p.q_rows * D;
            sdst_step = p.q_scale_pitch;
        } else {
            const int slot = p.ring ? p.ring->staged_slot[frame] : p.slot[frame];
            dst = p.kv_codes[tensor - 1] + ((size_t)slot * H * T + tok) * D;
            sdst = p.kv_scales[tensor - 1] + (size_t)slot * H * p.scale_pitch + tok;
            dst_step = (size_t)T * D;
            sdst_step = p.scale_pitch;
        }

        for (int h0 = 0; h0 < H; h0 += kItems) {
#pragma unroll
            for (int u = 0; u < kItems; ++u) {
                const int h = h0 + u;
                const HV ca = ra[u], cb = rb[u];
                if (row_ok && h + kItems < H) {
                    ra[u] = __ldcs(reinterpret_cast<const HV*>(item + (h + kItems) * D + ea));
                    rb[u] = __ldcs(reinterpret_cast<const HV*>(item + (h + kItems) * D + eb));
                }
                float xa[P], xb[P], ya[P], yb[P];
                unpack_bf16(ca, xa);
                unpack_bf16(cb, xb);
#pragma unroll
                for (int k = 0; k < P; ++k) {
                    const uint64_t t1 = fma2(pack2(xa[k], xb[k]), pack2(cc[k], cc[k]), mz2);
                    const uint64_t t2 = fma2(pack2(xb[k], xa[k]), pack2(-ss[k], ss[k]), mz2);
                    unpack2(fma2(t1, one2, t2), ya[k], yb[k]);
                }
                float amax = 0.f;
#pragma unroll
                for (int k = 0; k < P; ++k) amax = fmaxf(amax, fmaxf(fabsf(ya[k]), fabsf(yb[k])));
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (!row_ok || h >= H) continue;
                const bool keep = amax >= kMinAmax;
                const float inv = keep ? __fdiv_rn(448.f, amax) : 0.f;
                uint8_t* d = dst + (size_t)h * dst_step;
                if constexpr (P == 4) {
                    *reinterpret_cast<uint32_t*>(d + ea) =
                        e4m3x2(mul2(ya[0], ya[1], inv)) | ((uint32_t)e4m3x2(mul2(ya[2], ya[3], inv)) << 16);
                    *reinterpret_cast<uint32_t*>(d + eb) =
                        e4m3x2(mul2(yb[0], yb[1], inv)) | ((uint32_t)e4m3x2(mul2(yb[2], yb[3], inv)) << 16);
                } else {
                    *reinterpret_cast<uint16_t*>(d + ea) = e4m3x2(mul2(ya[0], ya[1], inv));
                    *reinterpret_cast<uint16_t*>(d + eb) = e4m3x2(mul2(yb[0], yb[1], inv));
                }
                if (lane16 == 0) sdst[(size_t)h * sdst_step] = keep ? div448(amax) : 0.f;
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 4) append_kernel(const __grid_constant__ AppendParams p)
{
    __shared__ unsigned int s_vmax[kMaxFrames][kMaxHeads];   // V only: largest scale per (frame, head)
    const int tensor = blockIdx.y;             // 0 = Q, 1 = K, 2 = V
    const int H = p.H;
#ifdef RTV_DEBUG
    // every staged frame must name a slot of the cache (the whole block returns alike)
    {
        bool bad = false;
        for (int f = 0; f < p.n_frames; ++f) {
            const int s = p.ring ? p.ring->staged_slot[f] : p.slot[f];
            bad |= s < 0 || s >= p.n_slots;
        }
        if (bad) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrBounds);
            return;
        }
    }
#endif
    if (tensor == 2) {
        for (int i = threadIdx.x; i < p.n_frames * H; i += kThreads) s_vmax[i / H][i % H] = 0u;
        __syncthreads();
        append_rows_v<D>(p, s_vmax);
        __syncthreads();
        const unsigned int seq = p.ring ? p.ring->seq : p.seq;
        for (int i = threadIdx.x; i < p.n_frames * H; i += kThreads) {
            const int f = i / H, h = i - f * H;
            const int slot = p.ring ? p.ring->staged_slot[f] : p.slot[f];
            const unsigned long long tag = ((unsigned long long)seq << 32) | s_vmax[f][h];
            atomicMax(&p.v_scale_max[(size_t)slot * H + h], tag);
        }
    } else {
        append_rows_rope<D>(p, tensor);
    }
}

// Blocks per tensor: one wave of the device (resident blocks per SM x SMs,
// shared by Q, K and V), or fewer when the chunk has fewer row groups.
template <int D>
cudaError_t blocks_per_tensor(int n_rows, int* out)
{
    static std::mutex mu;
    static int cap[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!cap[dev]) {
            int sms = 0, per_sm = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, append_kernel<D>, kThreads, 0);
            if (e != cudaSuccess) return e;
            cap[dev] = max(1, sms * max(1, per_sm) / 3);
        }
        *out = min(cap[dev], (n_rows + kGroups - 1) / kGroups);
    }
    return cudaSuccess;
}

template <int D>
cudaError_t launch(const AppendParams& p, cudaStream_t stream)
{
    int bx = 0;
    cudaError_t e = blocks_per_tensor<D>(p.n_frames * p.T, &bx);
    if (e != cudaSuccess) return e;
    append_kernel<D><<<dim3(bx, 3), kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t prepare_append(int D)
{
    int bx = 0;
    if (D == 128) return blocks_per_tensor<128>(1, &bx);
    if (D == 64) return blocks_per_tensor<64>(1, &bx);
    return cudaErrorInvalidValue;
}

cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t stream)
{
    if (D == 128) return launch<128>(p, stream);
    if (D == 64) return launch<64>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace rtv
