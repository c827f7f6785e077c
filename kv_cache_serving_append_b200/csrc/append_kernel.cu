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
// Work split: one block = up to rows_per_block token rows of one frame times
// all heads, for one of Q/K/V (blockIdx.y).  A (row, head) item is 2*D bytes
// of bf16, handled by a half-warp: each of the 16 lanes loads D/16 contiguous
// elements (16 bytes at D=128), so every input byte is read once with full
// 32-byte sectors, and writes D/16 codes (8 bytes), so the 16 lanes write one
// contiguous D-byte row of codes.  The rotate-half partner of a lane's
// elements sits 2 lanes away in the frame segment and 3 lanes away in the row
// and column segments (for the supported splits), fetched with a shuffle.
// Each group keeps ITEMS loads in flight to cover HBM latency.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "rtv_internal.h"

namespace rtv {
namespace {

constexpr int kThreads = 256;
constexpr int kGroups = kThreads / 16;   // half-warps per block
constexpr int kItems = 4;                // items in flight per half-warp

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

// E4M3 round-to-nearest-even with saturation to +-448 (hardware cvt).
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi)
{
    return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

template <int E>
__device__ __forceinline__ void store_codes(uint8_t* dst, const float* y, float inv);
template <>
__device__ __forceinline__ void store_codes<8>(uint8_t* dst, const float* y, float inv)
{
    uint32_t w0 = e4m3x2(__fmul_rn(y[0], inv), __fmul_rn(y[1], inv)) |
                  ((uint32_t)e4m3x2(__fmul_rn(y[2], inv), __fmul_rn(y[3], inv)) << 16);
    uint32_t w1 = e4m3x2(__fmul_rn(y[4], inv), __fmul_rn(y[5], inv)) |
                  ((uint32_t)e4m3x2(__fmul_rn(y[6], inv), __fmul_rn(y[7], inv)) << 16);
    *reinterpret_cast<uint2*>(dst) = make_uint2(w0, w1);
}
template <>
__device__ __forceinline__ void store_codes<4>(uint8_t* dst, const float* y, float inv)
{
    uint32_t w0 = e4m3x2(__fmul_rn(y[0], inv), __fmul_rn(y[1], inv)) |
                  ((uint32_t)e4m3x2(__fmul_rn(y[2], inv), __fmul_rn(y[3], inv)) << 16);
    *reinterpret_cast<uint32_t*>(dst) = w0;
}

constexpr int kMaxRows = 32;   // token rows per block (host keeps rows_per_block <= this)

template <int E>
__device__ __forceinline__ void load_vec(const float* p, float* x)
{
#pragma unroll
    for (int i = 0; i < E; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(p + i);
        x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
    }
}

__device__ __forceinline__ uint4 xor_vec(const uint4& v, uint32_t m) { return make_uint4(v.x ^ m, v.y ^ m, v.z ^ m, v.w ^ m); }
__device__ __forceinline__ uint2 xor_vec(const uint2& v, uint32_t m) { return make_uint2(v.x ^ m, v.y ^ m); }

// D = head_dim, E = D / 16 elements per lane.
template <int D>
__global__ void __launch_bounds__(kThreads, 4) append_kernel(const __grid_constant__ AppendParams p)
{
    constexpr int E = D / 16;
    using V = typename Vec<E>::T;
    // Per local token row: the RoPE cos/sin this row needs, laid out along
    // head_dim as [t cos | t sin | h cos | h sin | w cos | w sin] (half-widths).
    __shared__ __align__(16) float s_tab[kMaxRows][D];
    __shared__ unsigned int s_vmax[kMaxHeads];

    const int tensor = blockIdx.y;             // 0 = Q, 1 = K, 2 = V
    const int frame = blockIdx.x / p.blocks_per_frame;
    const int tok0 = (blockIdx.x % p.blocks_per_frame) * p.rows_per_block;
    const int n_rows = min(p.rows_per_block, p.T - tok0);
    const int H = p.H;
    const int n_items = n_rows * H;
    const bool rope = tensor != 2;
    const int ht = p.n_t / 2, hh = p.n_h / 2, hw = p.n_w / 2;

    for (int i = threadIdx.x; i < H; i += kThreads) s_vmax[i] = 0u;
    if (rope) {
        for (int i = threadIdx.x; i < n_rows * D; i += kThreads) {
            const int r = i / D, d = i - r * D;
            const int tok = tok0 + r;
            float v;
            if (d < 2 * ht) {
                v = p.t_table[frame][d / ht][d % ht];
            } else if (d < 2 * ht + 2 * hh) {
                const int hp = tok / p.grid_w;
                v = p.h_table[(size_t)hp * 2 * hh + (d - 2 * ht)];
            } else {
                const int wp = tok % p.grid_w;
                v = p.w_table[(size_t)wp * 2 * hw + (d - 2 * ht - 2 * hh)];
            }
            s_tab[r][d] = v;
        }
    }
    __syncthreads();

    const int lane16 = threadIdx.x & 15;
    const int group = threadIdx.x >> 4;
    const int lane = threadIdx.x & 31;

    // Fixed per lane: RoPE segment of its E elements, pair index of the
    // first one, which half of the pair it holds, its partner lane, and where
    // its cos/sin sit in the row table.
    int seg_half = ht, seg_lo = 0, tab_lo = 0;
    if (lane16 * E >= p.n_t + p.n_h) {
        seg_half = hw; seg_lo = p.n_t + p.n_h; tab_lo = 2 * ht + 2 * hh;
    } else if (lane16 * E >= p.n_t) {
        seg_half = hh; seg_lo = p.n_t; tab_lo = 2 * ht;
    }
    const int in_seg = lane16 * E - seg_lo;
    const bool first_half = in_seg < seg_half;
    const int j0 = first_half ? in_seg : in_seg - seg_half;
    const int partner = (lane & 16) | (first_half ? lane16 + seg_half / E : lane16 - seg_half / E);
    // x'[j] = x[j]c - x[j+n/2]s (first half) = x[j]c + (-x[j+n/2])s: the
    // partner's value is negated by flipping its bf16 sign bits (exact).
    const uint32_t neg_partner = first_half ? 0x80008000u : 0u;
    const int c_off = tab_lo + j0, s_off = tab_lo + seg_half + j0;

    const uint16_t* src = p.src[tensor];
    const int row0 = frame * p.T + tok0;

    // Item it = (row it / H, head it % H), visited with stride kGroups; the
    // (row, head) pair is advanced incrementally (no division per item).  The
    // loop bound is taken per warp so the full-warp shuffles always have all
    // 32 lanes present.
    int r_it = group / H, h_it = group - (group / H) * H;
    for (int wbase = group & ~1; wbase < n_items; wbase += kGroups * kItems) {
        const int base = wbase + (group & 1);
        V raw[kItems];
        int rr[kItems], hv[kItems];
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
            rr[u] = r_it;
            hv[u] = h_it;
            raw[u] = V{};
            if (base + u * kGroups < n_items) {
                const size_t off = ((size_t)(row0 + r_it) * H + h_it) * D + lane16 * E;
                raw[u] = __ldcs(reinterpret_cast<const V*>(src + off));
            }
            h_it += kGroups;
            while (h_it >= H) { h_it -= H; ++r_it; }
        }
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
            const bool valid = base + u * kGroups < n_items;
            const int r = valid ? rr[u] : 0;
            const int h = hv[u];
            float y[E];
            unpack_bf16(raw[u], y);
            if (rope) {
                const V praw = xor_vec(shfl_vec(raw[u], partner), neg_partner);
                float xp[E], cc[E], ss[E];
                unpack_bf16(praw, xp);
                load_vec<E>(&s_tab[r][c_off], cc);
                load_vec<E>(&s_tab[r][s_off], ss);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    y[e] = __fadd_rn(__fmul_rn(y[e], cc[e]), __fmul_rn(xp[e], ss[e]));
            }
            float amax = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[e]));
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            if (!valid) continue;
            const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
            const float scale = __fdiv_rn(amax, 448.f);
            const int tok = tok0 + r;
            uint8_t* dst;
            float* sdst;
            if (tensor == 0) {
                const size_t qr = (size_t)h * p.q_rows + frame * p.T + tok;
                dst = p.q_codes + qr * D;
                sdst = p.q_scales + (size_t)h * p.q_scale_pitch + frame * p.T + tok;
            } else {
                const size_t sh = (size_t)p.slot[frame] * H + h;
                dst = p.kv_codes[tensor - 1] + (sh * p.T + tok) * D;
                sdst = p.kv_scales[tensor - 1] + sh * p.scale_pitch + tok;
            }
            store_codes<E>(dst + lane16 * E, y, inv);
            if (lane16 == 0) {
                *sdst = scale;
                if (tensor == 2) atomicMax(&s_vmax[h], __float_as_uint(scale));
            }
        }
    }
    if (tensor == 2) {
        __syncthreads();
        for (int h = threadIdx.x; h < H; h += kThreads) {
            const unsigned long long tag = ((unsigned long long)p.seq << 32) | s_vmax[h];
            atomicMax(&p.v_scale_max[(size_t)p.slot[frame] * H + h], tag);
        }
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t stream)
{
    dim3 grid(p.n_frames * p.blocks_per_frame, 3);
    if (D == 128)
        append_kernel<128><<<grid, kThreads, 0, stream>>>(p);
    else if (D == 64)
        append_kernel<64><<<grid, kThreads, 0, stream>>>(p);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace rtv
