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
// row's heads.  A (row, head) item is 2*D bytes of bf16: lane i loads D/16
// contiguous elements (16 bytes at D = 128), so the 16 lanes read the item in
// full 32-byte sectors, and the H items of a row are one contiguous stretch
// of memory.  The RoPE cos/sin a lane needs depend only on the row (its
// frame, grid row and grid column) and on the lane's place in head_dim, so
// they are loaded into registers once per row and reused for every head.
// The rotate-half partner of a lane's elements sits 2 lanes away in the frame
// segment and 3 lanes away in the grid-row and grid-column segments (for the
// supported splits), fetched with a shuffle; the rotation's sign rides on the
// staged sine.  The arithmetic runs two elements per instruction where that
// is exact: the RoPE products and sum as f32x2 FMAs whose -0 addend and unit
// factor are kernel parameters (nothing the compiler could fold into a fused
// multiply-add), the quantising products as f32x2 multiplies, and the scale
// amax/448 as a product with the reciprocal corrected by its FMA residual.  Each half-warp keeps kItems
// loads in flight: the load of head h + kItems is issued as soon as head h is
// done.  Every input byte is read once and every code byte written once.
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
__device__ __forceinline__ uint4 shfl_vec(const uint4& v, int src)
{
    uint4 r;
    r.x = __shfl_sync(0xffffffffu, v.x, src);
    r.y = __shfl_sync(0xffffffffu, v.y, src);
    r.z = __shfl_sync(0xffffffffu, v.z, src);
    r.w = __shfl_sync(0xffffffffu, v.w, src);
    return r;
}
__device__ __forceinline__ uint2 shfl_vec(const uint2& v, int src)
{
    uint2 r;
    r.x = __shfl_sync(0xffffffffu, v.x, src);
    r.y = __shfl_sync(0xffffffffu, v.y, src);
    return r;
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

// amax / 448, correctly rounded: the product with RN(1/448) corrected once by
// its FMA residual (Markstein's correction step).  Checked against IEEE
// division for every positive finite float from 2^-120 up; below that (a
// subnormal quotient) the division itself is used.
__device__ __forceinline__ float div448(float a)
{
    if (!(a >= 0x1p-120f)) return __fdiv_rn(a, 448.f);
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

// E consecutive floats from a 16-byte aligned address.
template <int E>
__device__ __forceinline__ void load_vec(const float* p, float* x)
{
#pragma unroll
    for (int i = 0; i < E; i += 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p + i));
        x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
    }
}

// One tensor's rows (Q and K: ROPE; V: not rotated).  D = head_dim, E = D / 16
// elements per lane.
template <int D, bool ROPE>
__device__ __forceinline__ void append_rows(const AppendParams& p, int tensor,
                                            unsigned int (*s_vmax)[kMaxHeads], float* s_cs)
{
    constexpr int E = D / 16;
    using V = typename Vec<E>::T;
    constexpr bool rope = ROPE;
    const int H = p.H, T = p.T;
    const int n_rows = p.n_frames * T;
    const int ht = p.n_t / 2, hh = p.n_h / 2, hw = p.n_w / 2;

    const int lane16 = threadIdx.x & 15;
    const int lane = threadIdx.x & 31;

    // Fixed per lane: RoPE segment of its E elements (0 = frame, 1 = grid
    // row, 2 = grid column), pair index of the first one, which half of the
    // pair it holds, and its partner lane.
    int seg = 0, seg_half = ht, seg_lo = 0;
    if (lane16 * E >= p.n_t + p.n_h) {
        seg = 2; seg_half = hw; seg_lo = p.n_t + p.n_h;
    } else if (lane16 * E >= p.n_t) {
        seg = 1; seg_half = hh; seg_lo = p.n_t;
    }
    const int in_seg = lane16 * E - seg_lo;
    const bool first_half = in_seg < seg_half;
    const int j0 = first_half ? in_seg : in_seg - seg_half;
    const int partner = (lane & 16) | (first_half ? lane16 + seg_half / E : lane16 - seg_half / E);
    // x'[j] = x[j]c - x[j+n/2]s (first half) = x[j]c + x[j+n/2](-s): the sign
    // goes with the staged sine (fl(x(-s)) = -fl(xs) exactly).
    const float sin_sign = first_half ? -1.f : 1.f;

    const uint16_t* src = p.src[tensor];
    const uint64_t mz2 = pack2(p.neg_zero, p.neg_zero), one2 = pack2(p.one, p.one);
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

        // this lane's cos/sin for the row, staged in the half-warp's slice of
        // shared memory (read back per head; 16-byte accesses, no conflicts)
        // [cos | sin] x [e / 4][lane][4]: the 16 lanes' float4 accesses are consecutive
        float* cs = s_cs + ((threadIdx.x >> 4) * 2 * D) + lane16 * 4;   // cos at cs, sin at cs + D
        if (rope) {
            float cc[E], ss[E];
            if (seg == 0) {
                const float (*tt)[kMaxRopeHalf] = p.ring ? p.ring->t_table[frame] : p.t_table[frame];
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    cc[e] = tt[0][j0 + e];
                    ss[e] = tt[1][j0 + e];
                }
            } else if (seg == 1) {
                const float* t = p.h_table + (size_t)(tok / p.grid_w) * 2 * hh;
                load_vec<E>(t + j0, cc);
                load_vec<E>(t + hh + j0, ss);
            } else {
                const float* t = p.w_table + (size_t)(tok % p.grid_w) * 2 * hw;
                load_vec<E>(t + j0, cc);
                load_vec<E>(t + hw + j0, ss);
            }
            __syncwarp();   // the previous row's reads of this slice are done
#pragma unroll
            for (int e = 0; e < E; e += 4) {
                *reinterpret_cast<float4*>(cs + (e >> 2) * 64) = make_float4(cc[e], cc[e + 1], cc[e + 2], cc[e + 3]);
                *reinterpret_cast<float4*>(cs + D + (e >> 2) * 64) =
                    make_float4(sin_sign * ss[e], sin_sign * ss[e + 1], sin_sign * ss[e + 2], sin_sign * ss[e + 3]);
            }
            __syncwarp();
        }

        const V* item = reinterpret_cast<const V*>(src + (size_t)row * H * D + lane16 * E);
        V raw[kItems];
#pragma unroll
        for (int u = 0; u < kItems; ++u) raw[u] = (row_ok && u < H) ? __ldcs(item + (size_t)u * (D / E)) : V{};

        // destination of head 0 of this row, and the step from one head to the next
        uint8_t* dst;
        float* sdst;
        size_t dst_step, sdst_step;
        if (tensor == 0) {
            dst = p.q_codes + (size_t)row * D + lane16 * E;
            sdst = p.q_scales + row;
            dst_step = (size_t)p.q_rows * D;
            sdst_step = p.q_scale_pitch;
        } else {
            const int slot = p.ring ? p.ring->staged_slot[frame] : p.slot[frame];
            dst = p.kv_codes[tensor - 1] + ((size_t)slot * H * T + tok) * D + lane16 * E;
            sdst = p.kv_scales[tensor - 1] + (size_t)slot * H * p.scale_pitch + tok;
            dst_step = (size_t)T * D;
            sdst_step = p.scale_pitch;
        }

        for (int h0 = 0; h0 < H; h0 += kItems) {
#pragma unroll
            for (int u = 0; u < kItems; ++u) {
                const int h = h0 + u;
                const V cur = raw[u];
                // keep kItems loads in flight: the next load of this register
                if (row_ok && h + kItems < H) raw[u] = __ldcs(item + (size_t)(h + kItems) * (D / E));
                float y[E];
                unpack_bf16(cur, y);
                if (rope) {
                    const V praw = shfl_vec(cur, partner);
                    float xp[E], cc[E], ss[E];
                    unpack_bf16(praw, xp);
#pragma unroll
                    for (int e = 0; e < E; e += 4) {
                        const float4 c4 = *reinterpret_cast<const float4*>(cs + (e >> 2) * 64);
                        const float4 s4 = *reinterpret_cast<const float4*>(cs + D + (e >> 2) * 64);
                        cc[e] = c4.x; cc[e + 1] = c4.y; cc[e + 2] = c4.z; cc[e + 3] = c4.w;
                        ss[e] = s4.x; ss[e + 1] = s4.y; ss[e + 2] = s4.z; ss[e + 3] = s4.w;
                    }
                    // fl(fl(y c) + fl(xp s)), two elements per instruction: each
                    // product is an FMA with a -0 addend and the sum an FMA with a
                    // unit factor, both known only at run time (kernel parameters),
                    // so no step can be folded into a fused multiply-add and every
                    // operation rounds once, exactly as in the scalar form.
#pragma unroll
                    for (int e = 0; e < E; e += 2) {
                        const uint64_t t1 = fma2(pack2(y[e], y[e + 1]), pack2(cc[e], cc[e + 1]), mz2);
                        const uint64_t t2 = fma2(pack2(xp[e], xp[e + 1]), pack2(ss[e], ss[e + 1]), mz2);
                        unpack2(fma2(t1, one2, t2), y[e], y[e + 1]);
                    }
                }
                float amax = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[e]));
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (!row_ok || h >= H) continue;
                const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
                store_codes<E>(dst + (size_t)h * dst_step, y, inv);
                if (lane16 == 0) {
                    const float scale = div448(amax);
                    sdst[(size_t)h * sdst_step] = scale;
                    if (tensor == 2) atomicMax(&s_vmax[frame][h], __float_as_uint(scale));
                }
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 4) append_kernel(const __grid_constant__ AppendParams p)
{
    __shared__ unsigned int s_vmax[kMaxFrames][kMaxHeads];   // V only: largest scale per (frame, head)
    __shared__ __align__(16) float s_cs[kGroups * 2 * D];      // Q, K: per half-warp cos | sin of its row
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
        append_rows<D, false>(p, tensor, s_vmax, s_cs);
        __syncthreads();
        const unsigned int seq = p.ring ? p.ring->seq : p.seq;
        for (int i = threadIdx.x; i < p.n_frames * H; i += kThreads) {
            const int f = i / H, h = i - f * H;
            const int slot = p.ring ? p.ring->staged_slot[f] : p.slot[f];
            const unsigned long long tag = ((unsigned long long)seq << 32) | s_vmax[f][h];
            atomicMax(&p.v_scale_max[(size_t)slot * H + h], tag);
        }
    } else {
        append_rows<D, true>(p, tensor, s_vmax, s_cs);
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
