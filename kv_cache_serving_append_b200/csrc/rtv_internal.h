// rtv_internal.h -- launch parameter blocks shared by the host library and the
// kernels of librtv (never exposed through the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rtv.h"

namespace rtv {

constexpr int kMaxFrames = RTV_MAX_FRAMES_PER_CHUNK;
constexpr int kMaxSlots = RTV_MAX_SLOTS;
constexpr int kMaxHeads = 256;     // append kernel keeps one V-scale max per head in smem
constexpr int kMaxRopeHalf = 32;   // rope_t / 2 <= 32 (frame-axis table travels in params)

// Attention tiling shared by the kernel and the host-side TMA descriptors:
// 128 query rows per query tile, 64 keys per KV tile.
constexpr int kAttendRows = 128;
constexpr int kAttendKeys = 64;
constexpr int kMaxSplit = 4;       // key-range splits of one attention call
constexpr int kMaxDevices = 64;    // per-device one-time set-up tables

// Device error word bits.
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrBounds = 2u;    // debug builds: a kernel found a slot index out of range

// ------------------------------------------------------ device ring state --
// The ring state the kernels of a captured step graph read from device memory
// (in the cache buffer), so that one graph serves every step: the host
// uploads it when the graph is created (or when host calls moved the ring
// since), and the advance kernel at the end of each replayed step moves it
// one chunk forward.  Only the steady state is captured: the window is full
// (and the pinned frame committed), so the key set has a fixed frame count.
struct DeviceRing {
    // moved by the advance kernel
    long long G;                   // generated frames committed
    long long t0;                  // absolute frame index of staged frame 0
    unsigned int seq;              // V-scale-max tag of this step's appends
    int slot[kMaxSlots];           // key set, logical order: pinned, window, staged
    int staged_slot[kMaxFrames];
    float t_table[kMaxFrames][2][kMaxRopeHalf];   // frame-axis cos/sin of the staged frames
    // fixed for the life of a graph
    int n_staged, P0, C, W, n_keys, rope_half;
    double inv_freq[kMaxRopeHalf]; // rope_base^(-2j / rope_t), computed on the host
};

// ---------------------------------------------------------------- append --
struct AppendParams {
    const uint16_t* src[3];        // bf16 Q, K, V: [rows][H][D]
    uint8_t* q_codes;              // [H][q_rows][D]
    float* q_scales;               // [H][q_scale_pitch]
    uint8_t* kv_codes[2];          // K, V rings: [S][H][T][D]
    float* kv_scales[2];           // [S][H][scale_pitch]
    unsigned long long* v_scale_max;   // [S][H]
    const float* h_table;          // [grid_h][2][n_h/2]  (cos row, then sin row)
    const float* w_table;          // [grid_w][2][n_w/2]
    int H, D, T, grid_w, n_frames;
    int rows_per_block;            // token rows of one frame per block
    int blocks_per_frame;
    int q_rows;                    // F_max * T rows per head in the Q workspace
    int q_scale_pitch, scale_pitch;
    int n_t, n_h, n_w;
    unsigned int seq;              // append sequence number (V-scale max tag)
    int n_slots;                   // slots of the cache (debug builds check against it)
    unsigned int* err;             // device error word
    float neg_zero, one;           // -0.0f and 1.0f, as run-time values (see the RoPE in append_kernel.cu)
    int slot[kMaxFrames];          // ring slot of each staged frame
    float t_table[kMaxFrames][2][kMaxRopeHalf];   // frame-axis cos/sin per staged frame
    const DeviceRing* ring;        // non-null: take seq, slot and t_table from here
};

// ------------------------------------------------------------- attention --
struct AttendParams {
    const float* q_scales;         // [H][q_scale_pitch]
    const unsigned long long* v_scale_max;  // [S][H]
    void* out;                     // [M][H][D] fp32 or bf16
    unsigned int* err;             // device error word
    int H, D, T, M;                // M = n_frames * T query rows
    int q_scale_pitch;
    int out_bf16;
    int n_frames_keys;             // frames in the key set
    int key_tile;                  // keys per KV tile the tensor maps were encoded with (kAttendKeys)
    int tiles_per_frame;           // ceil(T / kAttendKeys)
    int n_split;                   // key-range splits (grid z); 1: no partials
    int tiles_per_split;           // KV tiles per split (the last may hold fewer)
    float* part_o;                 // [n_split][M][H][D] unnormalised O per split
    float* part_ml;                // [n_split][M][H][2] (reference exponent, row sum)
    int n_slots;                   // slots of the cache (debug builds check against it)
    int debug_wait_fault;          // 1: producer never arms the first barrier
    long long wait_limit;          // per-wait limit in clock cycles
    int slot[kMaxSlots];           // key set, logical order
    const DeviceRing* ring;        // non-null: take the key set's slots from here
};

// ----------------------------------------------- projection + append --
// x codes [R][Kd] E4M3 with s_x [R]; w codes [3*H*D][Kd] E4M3 with s_w [3*H*D]
// (rows: Q heads, then K heads, then V heads, each head's D features
// contiguous); the append part as for rtv_cache_append.
struct ProjectParams {
    AppendParams a;
    const float* sx;
    const float* sw;
    int R, Kd;
    int n_m_tiles, n_n_tiles;      // ceil(R / 128), 3*H*D / 256
    long long wait_limit;
    unsigned int* err;
};

// Launchers (defined in the .cu files).
cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t stream);
cudaError_t launch_attend(const AttendParams& p, const CUtensorMap* maps, int D,
                          cudaStream_t stream);
cudaError_t launch_ring_advance(DeviceRing* ring, cudaStream_t stream);
// One-time per-device launch set-up (attributes, occupancy), done before a
// stream capture so that none of it happens inside one.
cudaError_t prepare_append(int D);
cudaError_t prepare_attend(int D);
cudaError_t prepare_project();
cudaError_t launch_project(const ProjectParams& p, const CUtensorMap* maps, int sm_count,
                           cudaStream_t stream);
// maps: [0] Q codes, [1] K codes, [2] V codes, [3] K scales, [4] V scales

}  // namespace rtv
