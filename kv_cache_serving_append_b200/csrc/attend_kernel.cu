// attend_kernel.cu -- attention of a staged chunk over the ring-buffer KV cache:
// FP8 E4M3 QK^T and f16 PV on tcgen05 tensor cores with TMEM accumulators,
// online softmax in registers.
//
// Source of the operation: aidose.in, "Runway explains how it serves a 57B
// video model in real time", third paragraph (attention over the cache whose
// frames were rotated and quantised once, at write time); pttl.gr, section
// "Από οκτώ H100 σε τέσσερις" (240 attention calls per step).  The key set
// (pinned frame, window, chunk) and the 1/sqrt(D) softmax are the library's
// definition, stated in rtv.h.
//
// One CTA = two 128-row query tiles of one head, sharing every K/V tile it
// loads; KV tiles of 64 keys; 12 warps:
//   warp 0     TMA producer: both Q tiles once; per KV tile the K and V code
//              tiles at (ring slot * H + head, token tile) and their scales.
//   warps 1,3  MMA issuers, one per query tile t (warp 1 also owns TMEM).
//              S_t = Q_t K_j^T (kind::f8f6f4, E4M3 x E4M3 -> f32 in TMEM),
//              O_t += P_t,b V16_j (kind::f16, b = j mod 2, P read from TMEM,
//              V16 from shared memory).  S_t(j+2) is issued as soon as the
//              softmax has read S_t(j+1) into registers -- ahead of PV(j),
//              which is off the softmax's critical path -- so the next scores
//              are computed while the softmax works on the current ones.
//   warp 2     widens the V code tile to f16 (exact) in the MN-major layout
//              the PV MMA reads.
//   warps 4-7  softmax of query tile 0, warps 8-11 of query tile 1; one query
//              row per thread, the tile's 64 scores in registers, one pass
//              per KV tile against a reference m: s*scale_k, exp2, row sum,
//              P = p*scale_v/Sv in f16, kept in registers until the pass
//              stands and then stored to P_t,b in one TMEM store.  The row sum
//              bounds every p of the tile, so it alone decides (no per-key
//              max): a tile is redone against its exact max only when a row
//              sum reaches 2^15 (f16 P range), and m moves up by a power of
//              two, with O rescaled lazily, only when a row sum reaches 2^8.
//              The two warpgroups run concurrently.
// TMEM columns of query tile t: S_t [256t, 256t+64), P_t,0 and P_t,1 (f16
// pairs, 32 columns each) [256t+64, 256t+128), O_t [256t+128, 256t+128+D).
// S is single-buffered: QK(j+1) waits (s_free) until every softmax thread
// has read S(j).  P is double-buffered: softmax(j) writes P_t,b only after
// PV(j-2), its previous reader, has completed (pv_done).
// Per-tile waits avoid integer division (frame and tile-in-frame are walked),
// and at the end each warp's 32 output rows leave through shared memory so
// that the global stores write whole row segments.
//
// Logical-to-physical frame order is resolved in the TMA coordinates: the
// kernel receives the key set as a list of ring slots -- no gather, no copy.
//
// V's per-token scale varies along PV's contraction dimension, so it is
// folded into P.  Sv is a power of two at or above every V scale in the key
// set (from the per-frame V-scale maxima the append kernel records); P =
// p*scale_v/Sv stays below 2^15 (the redo bound), inside f16 range, and 1/Sv
// is folded into the exponent so the row sum carries the same factor and O/l
// needs none.
//
// When one CTA per (head, 256 query rows) would leave the last wave of the
// GPU mostly idle, the host splits every unit's key range (grid z); each split
// writes its unnormalised O and row statistics, and combine_kernel merges them.
//
// Registers: the block launches with 168 per thread; the four single-role
// warps give theirs back (setmaxnreg 56) and the softmax warps take them
// (setmaxnreg 224): 128 x 56 + 256 x 224 = 384 x 168.
//
// Every mbarrier wait is bounded; on time-out a thread sets the error word,
// leaves its loop, and the CTA drains its own async work before returning.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "rtv_internal.h"
#include "sm100.cuh"

namespace rtv {
namespace {

using namespace sm100;

constexpr int kBM = kAttendRows;   // query rows per query tile
constexpr int kQT = 2;             // query tiles per CTA
constexpr int kBN = kAttendKeys;   // keys per KV tile
constexpr int kStages = 6;         // K/V code tile stages
constexpr int kNV16 = 4;           // f16 V tile buffers
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr int kLazyRescaleLog2 = 8;     // move the reference when a tile's row sum reaches 2^8 of it
constexpr int kRedoLog2 = 15;           // redo a tile whose row sum reaches 2^15 (f16 P range)

__host__ __device__ constexpr uint32_t col_s(int t) { return 256u * t; }
__host__ __device__ constexpr uint32_t col_p(int t, int b) { return 256u * t + 64u + 32u * b; }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u * t + 128u; }

template <int D>
struct Smem {
    static constexpr int kQBytes = kBM * D;               // one FP8 query tile
    static constexpr int kKVBytes = kBN * D;              // one FP8 K or V tile
    static constexpr int kV16Bytes = kBN * D * 2;          // one f16 V tile
    alignas(1024) uint8_t q[kQT][kQBytes];
    alignas(1024) uint8_t k[kStages][kKVBytes];
    alignas(1024) uint8_t v8[kStages][kKVBytes];
    alignas(1024) uint8_t v16[kNV16][kV16Bytes];
    alignas(128) float sk[kStages][kBN];
    alignas(128) float sv[kStages][kBN];
    uint64_t q_full;
    uint64_t k_full[kStages];
    uint64_t kv_empty[kStages];
    uint64_t s_full[kQT], s_free[kQT], p_ready[kQT][2], pv_done[kQT][2];
    uint64_t v16_ready[kNV16], tile_done[kNV16];
    uint64_t drain[kQT];
    uint32_t tmem_base;
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction, two lanes of math).
__device__ __forceinline__ uint64_t pack2(float a, float b)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t r, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// Four E4M3 codes (bytes of w) -> four f16 (exact), as two packed pairs.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi)
{
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// Ring slot of frame f of the key set (from the device ring state when the
// launch belongs to a captured step graph).
__device__ __forceinline__ int key_slot(const AttendParams& p, int f)
{
    return p.ring ? p.ring->slot[f] : p.slot[f];
}

// Bounded wait whose outcome is the same for every lane of the warp, so that
// warp-collective tcgen05.ld/st never run with a partial warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, long long limit)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit));
}
__device__ __forceinline__ bool warp_wait_sleep(uint64_t* bar, uint32_t parity, long long limit)
{
    return __all_sync(0xffffffffu, mbar_wait_sleep(bar, parity, limit));
}

// Row max of u = s * scale_k over the valid keys of a KV tile (the kBN scores
// of this thread's row are in registers).  Used for the first KV tile and
// when a tile's scores outgrow the running max by more than f16 P allows.
template <bool kMask>
__device__ __forceinline__ float tile_row_max(const uint32_t* sr, const float* sk, int nv)
{
    const float4* sk4 = reinterpret_cast<const float4*>(sk);
    float mt[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int k4 = 0; k4 < kBN / 4; ++k4) {
        const float4 kk = sk4[k4];
        float a, b, c, d;
        unpack2(mul2(pack2(__uint_as_float(sr[4 * k4]), __uint_as_float(sr[4 * k4 + 1])),
                     pack2(kk.x, kk.y)), a, b);
        unpack2(mul2(pack2(__uint_as_float(sr[4 * k4 + 2]), __uint_as_float(sr[4 * k4 + 3])),
                     pack2(kk.z, kk.w)), c, d);
        float& m0 = mt[(k4 & 1) * 2];
        float& m1 = mt[(k4 & 1) * 2 + 1];
        if (!kMask) {
            m0 = max3(m0, a, b);
            m1 = max3(m1, c, d);
        } else {
            const int k = 4 * k4;
            if (k < nv) m0 = fmaxf(m0, a);
            if (k + 1 < nv) m1 = fmaxf(m1, b);
            if (k + 2 < nv) m0 = fmaxf(m0, c);
            if (k + 3 < nv) m1 = fmaxf(m1, d);
        }
    }
    return fmaxf(fmaxf(mt[0], mt[1]), fmaxf(mt[2], mt[3]));
}

// One pass over a KV tile (the kBN scores of this thread's row in registers):
// u = s * scale_k, x = u*c2 + neg (= (u - m)*c2 - log2 Sv for the reference
// m), p/Sv = 2^x, P = (p/Sv) * scale_v packed to f16 pairs in pk (key 2i and
// 2i+1 in pk[i]).  Nothing is stored: the caller writes P once it knows the
// pass stands and the P buffer is free, and the compiler is free to interleave
// the whole tile's exponentials.  Returns the row sum of p/Sv, which also
// bounds every p/Sv of the tile: the caller reads from it whether the tile
// outgrew m.
template <bool kMask>
__device__ __forceinline__ float tile_p(const uint32_t* sr, uint32_t* pk, const float* sk, const float* sv,
                                        uint64_t c2c2, uint64_t neg2, int nv)
{
    const float4* sk4 = reinterpret_cast<const float4*>(sk);
    const float4* sv4 = reinterpret_cast<const float4*>(sv);
    // independent partial row sums: short dependency chains
    uint64_t ls2[4] = {pack2(0.f, 0.f), pack2(0.f, 0.f), pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
    for (int k4 = 0; k4 < kBN / 4; ++k4) {
        const float4 kk = sk4[k4];
        const float4 vv = sv4[k4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int k = 4 * k4 + 2 * hh;
            const uint64_t u = mul2(pack2(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])),
                                    hh ? pack2(kk.z, kk.w) : pack2(kk.x, kk.y));
            float x0, x1;
            unpack2(fma2(u, c2c2, neg2), x0, x1);
            if (kMask) {
                if (k >= nv) x0 = -INFINITY;
                if (k + 1 >= nv) x1 = -INFINITY;
            }
            const float p0 = ex2(x0), p1 = ex2(x1);   // ex2(-inf) = 0 for masked keys
            const uint64_t pp = pack2(p0, p1);
            ls2[(k >> 1) & 3] = add2(ls2[(k >> 1) & 3], pp);
            float q0, q1;
            unpack2(mul2(pp, hh ? pack2(vv.z, vv.w) : pack2(vv.x, vv.y)), q0, q1);
            __half2 hv = __floats2half2_rn(q0, q1);
            pk[k / 2] = *reinterpret_cast<uint32_t*>(&hv);
        }
    }
    float a, b, c, d;
    unpack2(add2(ls2[0], ls2[1]), a, b);
    unpack2(add2(ls2[2], ls2[3]), c, d);
    return (a + b) + (c + d);
}

// TMEM store of 32 columns without a compiler memory clobber: it touches no
// generic memory, and its order against the tcgen05 waits, fences and
// mbarrier arrives (all volatile asm) is kept.
__device__ __forceinline__ void tmem_st32_p(uint32_t taddr, const uint32_t* r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

// Both phases complete (two try_waits in flight together), warp-uniform.
__device__ __forceinline__ bool warp_wait2(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb, long long limit)
{
    const bool ra = mbar_try_wait(a, pa);
    const bool rb = mbar_try_wait(b, pb);
    if (__all_sync(0xffffffffu, ra && rb)) return true;
    return __all_sync(0xffffffffu, mbar_wait(a, pa, limit) && mbar_wait(b, pb, limit));
}

__device__ __forceinline__ void reg_dealloc_56() { asm volatile("setmaxnreg.dec.sync.aligned.u32 56;"); }
__device__ __forceinline__ void reg_alloc_224() { asm volatile("setmaxnreg.inc.sync.aligned.u32 224;"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_kernel(const __grid_constant__ AttendParams p, const __grid_constant__ CUtensorMap map_q,
              const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
              const __grid_constant__ CUtensorMap map_sk, const __grid_constant__ CUtensorMap map_sv)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128B-swizzled tiles, by offsetting the
    // shared array itself (keeps the accesses in the shared address space)
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    Smem<D>& sm = *reinterpret_cast<Smem<D>*>(smem_raw + pad);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * (kQT * kBM);
    const int h = blockIdx.y;
    const int H = p.H;
    // this CTA's range of the key set: KV tiles [j0, j0 + n_tiles) (blockIdx.z = split)
    const int j0 = blockIdx.z * p.tiles_per_split;
    const int n_tiles = min(p.n_frames_keys * p.tiles_per_frame - j0, p.tiles_per_split);
    const int n_qt = min(kQT, (p.M - q0 + kBM - 1) / kBM);   // query tiles with valid rows
    const long long limit = p.wait_limit;
    // The K/V tensor maps' box must be this kernel's KV tile: a host built
    // against another tile size would have TMA write past the stage buffers.
    if (p.key_tile != kBN) {
        if (threadIdx.x == 0) atomicOr(p.err, kErrBounds);
        return;
    }
#ifdef RTV_DEBUG
    // every frame of the key set must name a slot of the cache: checked before
    // any barrier, TMEM or memory is touched; the whole CTA returns alike
    {
        bool bad = false;
        for (int f = 0; f < p.n_frames_keys; ++f) {
            const int s = key_slot(p, f);
            bad |= s < 0 || s >= p.n_slots;
        }
        if (bad) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrBounds);
            return;
        }
    }
#endif

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        // kv_empty / tile_done: one commit from each active query tile's issuer
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.kv_empty[s], n_qt);
        }
        for (int t = 0; t < kQT; ++t) {
            mbar_init(&sm.s_full[t], 1);
            mbar_init(&sm.s_free[t], 128);
            for (int b = 0; b < 2; ++b) {
                mbar_init(&sm.p_ready[t][b], 128);
                mbar_init(&sm.pv_done[t][b], 1);
            }
            mbar_init(&sm.drain[t], 1);
        }
        for (int b = 0; b < kNV16; ++b) {
            mbar_init(&sm.v16_ready[b], 32);
            mbar_init(&sm.tile_done[b], n_qt);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
        tma_prefetch_desc(&map_sk);
        tma_prefetch_desc(&map_sv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    bool fail = false;

    // setmaxnreg is executed by whole warpgroups (warps 0-3, 4-7, 8-11), as the
    // first instruction of each warpgroup's branch, so every region is
    // allocated by ptxas under the budget it runs with.
    if (warp < 4) {
        reg_dealloc_56();
        if (warp == 0) {
            // ------------------------------------------------------ producer --
            if (lane == 0 && !p.debug_wait_fault) {
                constexpr uint32_t kQBytes = Smem<D>::kQBytes, kKVBytes = Smem<D>::kKVBytes;
                mbar_arrive_expect_tx(&sm.q_full, kQT * kQBytes);
                for (int t = 0; t < kQT; ++t) tma_load_3d(sm.q[t], &map_q, &sm.q_full, 0, q0 + t * kBM, h);
                int issued = 0;
                int fi = j0 / p.tiles_per_frame, tif = j0 - fi * p.tiles_per_frame;
                for (int j = 0; j < n_tiles; ++j, tif = (tif + 1 == p.tiles_per_frame) ? (++fi, 0) : tif + 1) {
                    const int st = j % kStages;
                    if (j >= kStages &&
                        !mbar_wait_sleep(&sm.kv_empty[st], ((j / kStages) - 1) & 1, limit)) {
                        fail = true;
                        break;
                    }
                    const int t0 = tif * kBN;
                    const int row = key_slot(p, fi) * H + h;
                    mbar_arrive_expect_tx(&sm.k_full[st], 2 * kKVBytes + 2 * kBN * 4);
                    tma_load_3d(sm.k[st], &map_k, &sm.k_full[st], 0, t0, row);
                    tma_load_3d(sm.v8[st], &map_v, &sm.k_full[st], 0, t0, row);
                    tma_load_2d(sm.sk[st], &map_sk, &sm.k_full[st], t0, row);
                    tma_load_2d(sm.sv[st], &map_sv, &sm.k_full[st], t0, row);
                    ++issued;
                }
                // drain: every copy this thread issued has landed before the CTA may exit
                mbar_wait(&sm.q_full, 0, limit);
                for (int j = issued - kStages; j < issued; ++j) {
                    if (j < 0) continue;
                    mbar_wait(&sm.k_full[j % kStages], (j / kStages) & 1, limit);
                }
            }
        } else if (warp == 1 || warp == 3) {
            // ------------------------------------- MMA issuer of query tile t --
            const int t = warp == 1 ? 0 : 1;
            if (lane == 0 && t < n_qt) {
                constexpr uint32_t kQK = idesc(kBM, kBN, 0, 0, 0, 0);        // E4M3 x E4M3 -> f32
                constexpr uint32_t kPV = idesc(kBM, D, 0, 0, 0, 1);          // f16 x f16(MN) -> f32
                constexpr uint32_t kSw = D == 128 ? kSwizzle128 : kSwizzle64;
                constexpr uint32_t kSbo = D == 128 ? 1024 : 512;
                constexpr uint32_t kKVBytes = Smem<D>::kKVBytes, kV16Bytes = Smem<D>::kV16Bytes;
                // Descriptors are computed once: a buffer or K step only moves the
                // start-address field (bits 0-13, address >> 4; shared memory is
                // below 256 KB, so the add never carries out of the field).
                const uint64_t q_desc = smem_desc(smem_u32(sm.q[t]), 16, kSbo, kSw);
                const uint64_t k_desc0 = smem_desc(smem_u32(sm.k[0]), 16, kSbo, kSw);
                const uint64_t v_desc0 = smem_desc(smem_u32(sm.v16[0]), kBN * 128, 1024, kSwizzle128);
                // S_t = Q_t K_j^T once K_j has landed
                auto issue_qk = [&](int j) -> bool {
                    if (!mbar_wait_backoff(&sm.k_full[j % kStages], (j / kStages) & 1, limit)) return false;
                    tc_fence_after();
                    const uint64_t kd = k_desc0 + (uint64_t)(((j % kStages) * kKVBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk)
                        mma_f8_ss(tmem + col_s(t), q_desc + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2),
                                  kQK, kk > 0);
                    tc_commit(&sm.s_full[t]);
                    return true;
                };
                if (!mbar_wait_backoff(&sm.q_full, 0, limit)) fail = true;
                if (!fail && !issue_qk(0)) fail = true;
                // S(1) once every softmax thread has read S(0)
                if (!fail && n_tiles > 1 && (!mbar_wait(&sm.s_free[t], 0, limit) || !issue_qk(1))) fail = true;
                for (int j = 0; j < n_tiles && !fail; ++j) {
                    const int b = j & 1, vb = j % kNV16;
                    if (!mbar_wait(&sm.p_ready[t][b], (j >> 1) & 1, limit)) { fail = true; break; }
                    // S(j+2) as soon as softmax(j+1) has read S(j+1), ahead of PV(j):
                    // the next S is on the softmax's critical path, PV(j) is not
                    if (j + 2 < n_tiles) {
                        if (!mbar_wait(&sm.s_free[t], (j + 1) & 1, limit)) { fail = true; break; }
                        if (!issue_qk(j + 2)) { fail = true; break; }
                    }
                    // O_t += P_t,b V_j (P_b written by softmax(j), V_j widened)
                    if (!mbar_wait_backoff(&sm.v16_ready[vb], (j / kNV16) & 1, limit)) { fail = true; break; }
                    tc_fence_after();
                    const uint64_t vd = v_desc0 + (uint64_t)((vb * kV16Bytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk)
                        mma_f16_ts(tmem + col_o(t), tmem + col_p(t, b) + kk * 8, vd + (uint64_t)(kk * 128), kPV,
                                   (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&sm.pv_done[t][b]);
                    tc_commit(&sm.kv_empty[j % kStages]);
                    tc_commit(&sm.tile_done[vb]);
                }
                // drain: all MMAs issued by this thread complete before TMEM is freed
                tc_commit(&sm.drain[t]);
                if (!mbar_wait_backoff(&sm.drain[t], 0, limit)) fail = true;
            }
        } else if (warp == 2) {
            // ------------------------------------------- V widening (FP8->f16) --
            // A warp step covers 8 consecutive key rows x 4 chunk columns of one
            // 64-element block: in every 8-lane shared-memory phase the 8 rows hit
            // 8 different 16-byte bank groups, for the swizzled reads and for both
            // swizzled writes.
            constexpr int kNB = D / 64;                 // 64-element blocks per key row
            const int rl = lane & 7, cq = lane >> 3;
            // Lane (rl, cq) handles rows 8i + rl, 16-byte chunk nb*4 + cq of each: the
            // swizzle phase of those rows depends on rl only, so every address below
            // is a per-lane base plus a compile-time offset.
            const int sw = D == 128 ? rl : ((rl >> 1) & 3);
            int src_off[kNB];
#pragma unroll
            for (int nb = 0; nb < kNB; ++nb) src_off[nb] = rl * D + (((nb * 4 + cq) ^ sw) << 4);
            const int dst_a = rl * 128 + (((2 * cq) ^ rl) << 4);
            const int dst_b = rl * 128 + (((2 * cq + 1) ^ rl) << 4);
            for (int j = 0; j < n_tiles; ++j) {
                const int st = j % kStages, b = j % kNV16;
                if (!warp_wait_sleep(&sm.k_full[st], (j / kStages) & 1, limit)) { fail = true; break; }
                if (j >= kNV16 &&
                    !warp_wait_sleep(&sm.tile_done[b], ((j / kNV16) - 1) & 1, limit)) { fail = true; break; }
                const uint8_t* src = sm.v8[st];
                uint8_t* dst = sm.v16[b];
#pragma unroll 4
                for (int i = 0; i < kBN / 8; ++i) {
#pragma unroll
                    for (int nb = 0; nb < kNB; ++nb) {
                        const uint4 raw = *reinterpret_cast<const uint4*>(src + src_off[nb] + i * 8 * D);
                        uint32_t o[8];
                        e4m3x4_to_f16x4(raw.x, o[0], o[1]);
                        e4m3x4_to_f16x4(raw.y, o[2], o[3]);
                        e4m3x4_to_f16x4(raw.z, o[4], o[5]);
                        e4m3x4_to_f16x4(raw.w, o[6], o[7]);
                        // elements 16c .. 16c+15 (c = nb*4 + cq) = bytes 32*cq .. 32*cq+31 of block nb's row
                        uint8_t* rowp = dst + nb * (kBN * 128) + i * 8 * 128;
                        *reinterpret_cast<uint4*>(rowp + dst_a) = make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4*>(rowp + dst_b) = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
                fence_async_smem();   // generic-proxy writes -> visible to the MMA's async proxy
                mbar_arrive(&sm.v16_ready[b]);
            }
        }
    } else {
        // --------------------------------------------------------- softmax --
        reg_alloc_224();
        const int t = (warp - 4) >> 2;              // query tile of this warpgroup
        if (t < n_qt) {
            const int row = (warp & 3) * 32 + lane;     // TMEM lane == query row in tile
            const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
            const uint32_t t_o = tmem + lane_off + col_o(t);
            const int qrow = q0 + t * kBM + row;
            const bool row_ok = qrow < p.M;
            const float sq = row_ok ? p.q_scales[(size_t)h * p.q_scale_pitch + qrow] : 0.f;
            constexpr float kInvSqrtD = D == 128 ? 0.08838834764831845f : 0.125f;
            const float c2 = sq * (1.4426950408889634f * kInvSqrtD);   // log2(e) / sqrt(D) * scale_q

            // Sv: power of two >= every V scale of the key set
            float vmax = 0.f;
            for (int f = lane; f < p.n_frames_keys; f += 32)
                vmax = fmaxf(vmax, __uint_as_float((uint32_t)(
                                       p.v_scale_max[(size_t)key_slot(p, f) * H + h] & 0xffffffffull)));
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
            int ve = (int)((__float_as_uint(vmax) >> 23) & 0xff);
            if (__float_as_uint(vmax) & 0x7fffff) ve += 1;
            if (!(vmax > 0.f)) ve = 127;
            ve = max(127 - 60, min(127 + 60, ve));
            const float log2_sv = (float)(ve - 127);

            float m = 0.f;         // reference of s * scale_k (the max of KV tile 0, moved up lazily)
            float l = 0.f;         // running sum of p / Sv, relative to m
            float o_scale = 1.f;   // factor O still owes (applied before the next PV)
            const uint64_t c2c2 = pack2(c2, c2);
            const int log2_sv_i = ve - 127;
            const uint32_t t_s = tmem + lane_off + col_s(t);
            int tif = j0 % p.tiles_per_frame;       // KV tile index within its frame
            for (int j = 0; j < n_tiles && !fail; ++j, tif = (tif + 1 == p.tiles_per_frame) ? 0 : tif + 1) {
                const int st = j % kStages, b = j & 1;
                const int nv = min(kBN, p.T - tif * kBN);
                const uint32_t t_p = tmem + lane_off + col_p(t, b);
                if (!warp_wait2(&sm.k_full[st], (j / kStages) & 1, &sm.s_full[t], j & 1, limit)) { fail = true; break; }
                tc_fence_after();
                uint32_t sr[kBN];
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) tmem_ld32(t_s + c * 32, sr + c * 32);
                tc_wait_ld();
                // S is in registers: the issuer may overwrite it with the next tile's scores
                tc_fence_before();
                mbar_arrive(&sm.s_free[t]);
                // P_b was last read by PV(j-2): tested now, waited for only
                // before the P store, so the test's latency hides behind the pass
                const bool p_free = j < 2 || mbar_test(&sm.pv_done[t][b], ((j - 2) >> 1) & 1);
                if (j == 0)   // the first tile sets the reference
                    m = nv == kBN ? tile_row_max<false>(sr, sm.sk[st], nv)
                                  : tile_row_max<true>(sr, sm.sk[st], nv);
                // single pass against the reference: p/Sv = 2^(u*c2 - m*c2 - log2 Sv).
                // The row sum bounds every p of the tile; if some row's sum
                // (times Sv) reaches 2^15, a p may be past f16 P range and the
                // pass is redone once against the tile's exact max (rare: the
                // first tiles of a row).  ls_e = floor(log2(row sum * Sv)).
                float ls = 0.f;
                int ls_e = 0;
                uint32_t pk[kBN / 2];
#pragma unroll 1
                for (int attempt = 0; attempt < 2; ++attempt) {
                    const float neg = -(m * c2 + log2_sv);
                    ls = nv == kBN ? tile_p<false>(sr, pk, sm.sk[st], sm.sv[st], c2c2, pack2(neg, neg), nv)
                                   : tile_p<true>(sr, pk, sm.sk[st], sm.sv[st], c2c2, pack2(neg, neg), nv);
                    ls_e = (int)((__float_as_uint(ls) >> 23) & 0xff) - 127 + log2_sv_i;
                    if (attempt == 1 || !__any_sync(0xffffffffu, ls_e >= kRedoLog2)) break;
                    const float mt = nv == kBN ? tile_row_max<false>(sr, sm.sk[st], nv)
                                               : tile_row_max<true>(sr, sm.sk[st], nv);
                    const float m_new = fmaxf(m, mt);
                    const float alpha = ex2((m - m_new) * c2);
                    l *= alpha;
                    o_scale *= alpha;
                    m = m_new;
                }
                l += ls;
                if (!__all_sync(0xffffffffu, p_free) &&
                    !warp_wait(&sm.pv_done[t][b], ((j - 2) >> 1) & 1, limit)) { fail = true; break; }
                tc_fence_after();
                tmem_st32_p(t_p, pk);
                // O owes a factor from an earlier move of m: apply it once PV(j-1)
                // has completed and before PV(j) is issued (warp-uniform: the
                // wait and the TMEM load/store are warp-collective).
                if (__any_sync(0xffffffffu, o_scale != 1.f)) {
                    if (j > 0 && !warp_wait(&sm.pv_done[t][(j - 1) & 1], ((j - 1) >> 1) & 1, limit)) { fail = true; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(t_o + c * 32, o);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * o_scale);
                        tmem_st32(t_o + c * 32, o);
                    }
                    o_scale = 1.f;
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.p_ready[t][b]);
                // lazy move of the reference: only when this tile's row sum grew
                // to 2^8 of it; by an exact power of two, l now, O before the next
                // PV (after PV(j)).
                if (ls_e >= kLazyRescaleLog2) {
                    const float alpha = __uint_as_float((uint32_t)(127 - ls_e) << 23);   // 2^-ls_e
                    l *= alpha;
                    o_scale *= alpha;
                    m += (float)ls_e / c2;
                }
            }
            if (!fail && !warp_wait(&sm.pv_done[t][(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, limit))
                fail = true;
            if (!fail) {
                tc_fence_after();
                // one split: the normalised output.  Several: this range's O
                // (owed factor applied, not normalised) and its row statistics
                // (reference exponent m*c2, row sum l), merged by the combine
                // kernel.
                const bool split = p.n_split > 1;
                const size_t part_row = ((size_t)blockIdx.z * p.M + qrow) * H + h;
                if (split && row_ok)
                    *reinterpret_cast<float2*>(p.part_ml + 2 * part_row) = make_float2(m * c2, l);
                const float norm = split ? o_scale : o_scale / l;
                // The warp's 32 rows leave through shared memory so that every
                // global store writes whole row segments (4 rows x 128 bytes per
                // instruction instead of 32 scattered 16-byte pieces).  The staging
                // buffer is this query tile's Q code tile: its last reader, QK of
                // the last KV tile, completed before PV of that tile did.
                constexpr int kCW = Smem<D>::kQBytes / (4 * 32 * 4);   // staged columns per pass: 32 (D128), 16 (D64)
                constexpr int kG = kCW / 4;                              // float4 groups per staged row
                constexpr int kRpi = 32 / kG;                            // rows per warp store instruction
                float* stg = reinterpret_cast<float*>(sm.q[t]) + (warp & 3) * (32 * kCW);
                const int qbase = q0 + t * kBM + (warp & 3) * 32;
                const bool bf = p.out_bf16 && !split;
                const int gl = lane % kG;                                // float4 group this lane stores
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_o + c * 32, o);
                    tc_wait_ld();
#pragma unroll
                    for (int hc = 0; hc < 32 / kCW; ++hc) {
                        // row `lane` of the pass: float4 group g at slot g ^ (lane mod kG)
#pragma unroll
                        for (int g = 0; g < kG; ++g) {
                            const int e = hc * kCW + 4 * g;
                            *reinterpret_cast<float4*>(stg + lane * kCW + 4 * (g ^ (lane % kG))) =
                                make_float4(__uint_as_float(o[e]) * norm, __uint_as_float(o[e + 1]) * norm,
                                            __uint_as_float(o[e + 2]) * norm, __uint_as_float(o[e + 3]) * norm);
                        }
                        __syncwarp();
#pragma unroll
                        for (int it = 0; it < kG; ++it) {
                            const int r = it * kRpi + lane / kG;
                            const float4 v = *reinterpret_cast<const float4*>(stg + r * kCW + 4 * (gl ^ (r % kG)));
                            const int qr = qbase + r;
                            if (qr < p.M) {
                                const int col = c * 32 + hc * kCW + 4 * gl;
                                if (bf) {
                                    __nv_bfloat162 a2 = __floats2bfloat162_rn(v.x, v.y);
                                    __nv_bfloat162 b2 = __floats2bfloat162_rn(v.z, v.w);
                                    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) +
                                                              ((size_t)qr * H + h) * D + col) =
                                        make_uint2(*reinterpret_cast<uint32_t*>(&a2), *reinterpret_cast<uint32_t*>(&b2));
                                } else {
                                    float* dst = split ? p.part_o + (((size_t)blockIdx.z * p.M + qr) * H + h) * D
                                                       : reinterpret_cast<float*>(p.out) + ((size_t)qr * H + h) * D;
                                    *reinterpret_cast<float4*>(dst + col) = v;
                                }
                            }
                        }
                        __syncwarp();
                    }
                }
            }
        }
    }

    if (fail) atomicOr(p.err, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge of the key-range splits: one warp per (query row, head).  Split s
// holds O_s = sum_{keys in s} 2^(x - e_s) v (unnormalised) and l_s = sum 2^(x
// - e_s) against its own reference exponent e_s; out = sum_s 2^(e_s - e) O_s
// / sum_s 2^(e_s - e) l_s with e = max_s e_s (the online-softmax merge).  The
// split count is a template parameter, so every split's loads are in flight
// together.
static_assert(kMaxSplit >= 2 && kMaxSplit <= 4, "combine_kernel is instantiated for 2, 3 and 4 splits");
template <int D, int S>
__global__ void __launch_bounds__(256) combine_kernel(const AttendParams p)
{
    const int warp = (blockIdx.x * 256 + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= p.M * p.H) return;
    const size_t stride = (size_t)p.M * p.H;          // rows of one split
    constexpr int kV = D / 32;                          // elements per lane
    float2 ml[S];
    float v[S][kV];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        ml[s] = *reinterpret_cast<const float2*>(p.part_ml + 2 * (s * stride + warp));
        const float* src = p.part_o + (s * stride + warp) * D + lane * kV;
        if constexpr (kV == 4) {
            const float4 x = __ldcs(reinterpret_cast<const float4*>(src));
            v[s][0] = x.x; v[s][1] = x.y; v[s][2] = x.z; v[s][3] = x.w;
        } else {
            const float2 x = __ldcs(reinterpret_cast<const float2*>(src));
            v[s][0] = x.x; v[s][1] = x.y;
        }
    }
    float e = -INFINITY;
#pragma unroll
    for (int s = 0; s < S; ++s) e = fmaxf(e, ml[s].x);
    float acc[kV] = {};
    float lsum = 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const float w = exp2f(ml[s].x - e);
        lsum += w * ml[s].y;
#pragma unroll
        for (int i = 0; i < kV; ++i) acc[i] += w * v[s][i];
    }
    const float inv = 1.f / lsum;
    if (p.out_bf16) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)warp * D + lane * kV;
#pragma unroll
        for (int i = 0; i < kV; i += 2)
            *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
    } else {
        float* dst = reinterpret_cast<float*>(p.out) + (size_t)warp * D + lane * kV;
        if constexpr (kV == 4)
            __stcs(reinterpret_cast<float4*>(dst), make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv));
        else
            __stcs(reinterpret_cast<float2*>(dst), make_float2(acc[0] * inv, acc[1] * inv));
    }
}

// Raise the kernel's dynamic shared-memory limit once per device (the
// attribute is per device and per function); guarded for concurrent callers.
template <int D>
cudaError_t configure_once(int dev, size_t smem)
{
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

template <int D>
cudaError_t launch(const AttendParams& p, const CUtensorMap* maps, cudaStream_t stream)
{
    const size_t smem = sizeof(Smem<D>) + 1024;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = configure_once<D>(dev, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.M + kQT * kBM - 1) / (kQT * kBM), p.H, p.n_split);
    attend_kernel<D><<<grid, kThreads, smem, stream>>>(p, maps[0], maps[1], maps[2], maps[3], maps[4]);
    if (p.n_split > 1) {
        const long long warps = (long long)p.M * p.H;
        const unsigned blocks = (unsigned)((warps + 7) / 8);
        switch (p.n_split) {
            case 2: combine_kernel<D, 2><<<blocks, 256, 0, stream>>>(p); break;
            case 3: combine_kernel<D, 3><<<blocks, 256, 0, stream>>>(p); break;
            default: combine_kernel<D, 4><<<blocks, 256, 0, stream>>>(p); break;
        }
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t prepare_attend(int D)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (D == 128) return configure_once<128>(dev, sizeof(Smem<128>) + 1024);
    if (D == 64) return configure_once<64>(dev, sizeof(Smem<64>) + 1024);
    return cudaErrorInvalidValue;
}

cudaError_t launch_attend(const AttendParams& p, const CUtensorMap* maps, int D, cudaStream_t stream)
{
    if (D == 128) return launch<128>(p, maps, stream);
    if (D == 64) return launch<64>(p, maps, stream);
    return cudaErrorInvalidValue;
}

}  // namespace rtv
