// project_kernel.cu -- the QKV projection as an FP8 GEMM on tcgen05 tensor
// cores with the cache append fused into its epilogue: the bf16 Q/K/V never
// travel through HBM.
//
// Source: lhc.media, "Runway partage la construction de Runway Characters",
// third paragraph (matmul and kernel tuning); aidose.in, "Runway explains how
// it serves a 57B video model in real time", third paragraph (FP8 matmuls;
// rotary embedding and FP8 quantisation applied once, as a frame enters the
// cache).  The projection's inputs are E4M3 codes with one fp32 scale per
// token row (activations) and per output channel (weights); its output, the
// bf16 Q/K/V the append consumes, is
//     qkv[r][n] = bf16_rne( fl( fl(acc[r][n] * s_x[r]) * s_w[n] ) ),
//     acc[r][n] = sum_k decode(x[r][k]) * decode(w[n][k])  (fp32 accumulate),
// and the epilogue then applies exactly the append's arithmetic (3D RoPE on
// Q and K, amax, scale, E4M3) to each (row, head) of it.
//
// Tiles: 128 token rows x 256 output features (two heads of one of Q/K/V), K
// in steps of 128 codes (one 128-byte swizzled row per operand row).  The
// kernel is persistent: each CTA walks tiles n-major (CTAs running at the
// same time share weight tiles in L2).  Warps:
//   warp 0     TMA producer: A (x) and B (w) tiles into a 4-stage ring.
//   warp 1     MMA issuer: kind::f8f6f4 M=128 N=256 K=32, into one of two
//              TMEM accumulators of 256 columns (TMEM owner).
//   warps 2-5  epilogue: one token row per thread, reading its 2 x 128 fp32
//              accumulators from TMEM while the MMAs of the next tile run
//              into the other accumulator.
// RoPE here is specialised to head_dim 128 split t:h:w = 32:48:48 (the
// host rejects other shapes for this entry point).  Every mbarrier wait is
// bounded; on time-out the error word is set and the CTA drains and exits.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "rtv_internal.h"
#include "sm100.cuh"

namespace rtv {
namespace {

using namespace sm100;

constexpr int kPM = 128;          // token rows per tile
constexpr int kPN = 256;          // output features per tile (two heads)
constexpr int kPK = 128;          // codes per K step (128 bytes)
constexpr int kPStages = 4;
constexpr int kPThreads = 192;
constexpr int kD = 128;           // head_dim of the fused path
constexpr int kNT = 32, kNH = 48, kNW = 48;   // RoPE split of the fused path

struct ProjSmem {
    alignas(1024) uint8_t a[kPStages][kPM * kPK];
    alignas(1024) uint8_t b[kPStages][kPN * kPK];
    uint64_t full[kPStages], empty[kPStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
};

// One (row, head) item: 128 projected values in registers -> RoPE (Q, K) ->
// amax -> E4M3 codes and scale, written where the append writes them.
__device__ __forceinline__ void quantise_store(float (&y)[kD], bool rope, const float* cs_t,
                                               const float* cs_h, const float* cs_w, uint8_t* dst,
                                               float* sdst, float* scale_out)
{
    if (rope) {
        // rotate-half within each segment: x'[j] = x[j]c - x[j+n/2]s,
        // x'[j+n/2] = x[j+n/2]c + x[j]s, one rounding per operation
#pragma unroll
        for (int j = 0; j < kNT / 2; ++j) {
            const float c = cs_t[j], s = cs_t[kNT / 2 + j];
            const float a = y[j], b = y[j + kNT / 2];
            y[j] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
            y[j + kNT / 2] = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
        }
#pragma unroll
        for (int j = 0; j < kNH / 2; ++j) {
            const float c = cs_h[j], s = cs_h[kNH / 2 + j];
            const float a = y[kNT + j], b = y[kNT + j + kNH / 2];
            y[kNT + j] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
            y[kNT + j + kNH / 2] = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
        }
#pragma unroll
        for (int j = 0; j < kNW / 2; ++j) {
            const float c = cs_w[j], s = cs_w[kNW / 2 + j];
            const float a = y[kNT + kNH + j], b = y[kNT + kNH + j + kNW / 2];
            y[kNT + kNH + j] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
            y[kNT + kNH + j + kNW / 2] = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
        }
    }
    float amax = 0.f;
#pragma unroll
    for (int d = 0; d < kD; ++d) amax = fmaxf(amax, fabsf(y[d]));
    // below 2^-119 the reciprocal would overflow: such an item is stored as zero
    const bool keep = amax >= 0x1p-119f;
    const float inv = keep ? __fdiv_rn(448.f, amax) : 0.f;
    const float scale = keep ? __fdiv_rn(amax, 448.f) : 0.f;
#pragma unroll
    for (int c = 0; c < kD / 16; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = 16 * c + 4 * e;
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(y[d], inv), __fmul_rn(y[d + 1], inv)),
                                                         __NV_SATFINITE, __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(y[d + 2], inv), __fmul_rn(y[d + 3], inv)),
                                                         __NV_SATFINITE, __NV_E4M3);
            w[e] = (lo & 0xffffu) | (hi << 16);
        }
        if (dst) *reinterpret_cast<uint4*>(dst + 16 * c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (sdst) *sdst = scale;
    *scale_out = scale;
}

__global__ void __launch_bounds__(kPThreads, 1)
project_kernel(const __grid_constant__ ProjectParams p, const __grid_constant__ CUtensorMap map_x,
               const __grid_constant__ CUtensorMap map_w)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    ProjSmem& sm = *reinterpret_cast<ProjSmem*>(smem_raw + pad);
    const AppendParams& a = p.a;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = p.n_m_tiles * p.n_n_tiles;
    const int k_steps = p.Kd / kPK;
    const long long limit = p.wait_limit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 4);
        }
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    bool fail = false;

    if (warp == 0) {
        // ---------------------------------------------------------- producer --
        if (lane == 0) {
            int it = 0, issued = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !fail; tile += gridDim.x) {
                const int mt = tile % p.n_m_tiles, nt = tile / p.n_m_tiles;
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const int st = it % kPStages;
                    if (it >= kPStages &&
                        !mbar_wait_sleep(&sm.empty[st], ((it / kPStages) - 1) & 1, limit)) {
                        fail = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[st], (kPM + kPN) * kPK);
                    tma_load_2d(sm.a[st], &map_x, &sm.full[st], ks * kPK, mt * kPM);
                    tma_load_2d(sm.b[st], &map_w, &sm.full[st], ks * kPK, nt * kPN);
                    ++issued;
                }
            }
            for (int j = issued - kPStages; j < issued; ++j)   // drain: copies land before exit
                if (j >= 0) mbar_wait(&sm.full[j % kPStages], (j / kPStages) & 1, limit);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer --
        if (lane == 0) {
            constexpr uint32_t kId = idesc(kPM, kPN, 0, 0, 0, 0);   // E4M3 x E4M3 -> f32
            int it = 0, local = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !fail; tile += gridDim.x, ++local) {
                const int buf = local & 1;
                if (local >= 2 && !mbar_wait_backoff(&sm.acc_empty[buf], ((local / 2) - 1) & 1, limit)) {
                    fail = true;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const int st = it % kPStages;
                    if (!mbar_wait_backoff(&sm.full[st], (it / kPStages) & 1, limit)) { fail = true; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sm.a[st]), b_addr = smem_u32(sm.b[st]);
#pragma unroll
                    for (int kk = 0; kk < kPK / 32; ++kk)
                        mma_f8_ss(tmem + buf * kPN, smem_desc(a_addr + kk * 32, 16, 1024, kSwizzle128),
                                  smem_desc(b_addr + kk * 32, 16, 1024, kSwizzle128), kId,
                                  (ks > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&sm.empty[st]);
                }
                if (fail) break;
                tc_commit(&sm.acc_full[buf]);
            }
            tc_commit(&sm.drain);
            if (!mbar_wait_backoff(&sm.drain, 0, limit)) fail = true;
        }
    } else {
        // ---------------------------------------------------------- epilogue --
        const int q = warp & 3;                          // TMEM lane quarter of this warp
        const int row = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const int HD = a.H * kD;
        int local = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++local) {
            const int buf = local & 1;
            const int mt = tile % p.n_m_tiles, nt = tile / p.n_m_tiles;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[buf], (local / 2) & 1, limit))) {
                fail = true;
                break;
            }
            tc_fence_after();
            const int r = mt * kPM + row;                // token row of the chunk
            const bool ok = r < p.R;
            const int frame = ok ? r / a.T : 0, tok = ok ? r - frame * a.T : 0;
            const float sx = ok ? p.sx[r] : 0.f;
            const int n0 = nt * kPN;
            const int tensor = n0 / HD;                  // both heads of a tile: one tensor
            const bool rope = tensor != 2;
            const int slot = tensor == 0 ? 0 : (a.ring ? a.ring->staged_slot[frame] : a.slot[frame]);
            // this row's RoPE cos/sin: [cos | sin] per segment
            const float* cs_t = a.ring ? &a.ring->t_table[frame][0][0] : &a.t_table[frame][0][0];
            float ct[kNT];
#pragma unroll
            for (int j = 0; j < kNT / 2; ++j) {
                ct[j] = cs_t[j];
                ct[kNT / 2 + j] = cs_t[kMaxRopeHalf + j];
            }
            const float* ch = a.h_table + (size_t)(tok / a.grid_w) * kNH;
            const float* cw = a.w_table + (size_t)(tok % a.grid_w) * kNW;
            for (int hh = 0; hh < 2; ++hh) {
                const int n = n0 + hh * kD;
                const int head = (n - tensor * HD) / kD;
                float y[kD];
#pragma unroll
                for (int c = 0; c < kD / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_off + buf * kPN + hh * kD + c * 32, v);
                    tc_wait_ld();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 w4 = __ldg(reinterpret_cast<const float4*>(p.sw + n + c * 32 + 4 * i4));
                        const float ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 4 * i4 + e;
                            const float t = __fmul_rn(__fmul_rn(__uint_as_float(v[i]), sx), ws[e]);
                            y[c * 32 + i] = __bfloat162float(__float2bfloat16_rn(t));
                        }
                    }
                }
                // rows past the chunk (zero-filled by TMA) are computed but not stored
                uint8_t* dst = nullptr;
                float* sdst = nullptr;
                if (tensor == 0) {
                    dst = a.q_codes + ((size_t)head * a.q_rows + r) * kD;
                    sdst = a.q_scales + (size_t)head * a.q_scale_pitch + r;
                } else {
                    const size_t sh = (size_t)slot * a.H + head;
                    dst = a.kv_codes[tensor - 1] + (sh * a.T + tok) * kD;
                    sdst = a.kv_scales[tensor - 1] + sh * a.scale_pitch + tok;
                }
                float scale = 0.f;
                quantise_store(y, rope, ct, ch, cw, ok ? dst : nullptr, ok ? sdst : nullptr, &scale);
                if (tensor == 2) {
                    // largest V scale per (frame, head) over the warp's rows (one
                    // frame at a time; all 32 lanes take part), one tag per frame
                    const unsigned int seq = a.ring ? a.ring->seq : a.seq;
                    bool done = !ok;
                    while (__any_sync(0xffffffffu, !done)) {
                        const int f = __reduce_min_sync(0xffffffffu, done ? 0x7fffffff : frame);
                        float m = (!done && frame == f) ? scale : 0.f;
#pragma unroll
                        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        if (lane == 0) {
                            const int fs = a.ring ? a.ring->staged_slot[f] : a.slot[f];
                            atomicMax(&a.v_scale_max[(size_t)fs * a.H + head],
                                      ((unsigned long long)seq << 32) | __float_as_uint(m));
                        }
                        if (frame == f) done = true;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
        }
    }

    if (fail) atomicOr(p.err, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t prepare_project()
{
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        e = cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(sizeof(ProjSmem) + 1024));
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

cudaError_t launch_project(const ProjectParams& p, const CUtensorMap* maps, int sm_count, cudaStream_t stream)
{
    cudaError_t e = prepare_project();
    if (e != cudaSuccess) return e;
    const int tiles = p.n_m_tiles * p.n_n_tiles;
    project_kernel<<<min(tiles, sm_count), kPThreads, sizeof(ProjSmem) + 1024, stream>>>(p, maps[0], maps[1]);
    return cudaGetLastError();
}

}  // namespace rtv
