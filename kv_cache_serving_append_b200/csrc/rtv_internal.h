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
    int slot[kMaxFrames];          // ring slot of each staged frame
    float t_table[kMaxFrames][2][kMaxRopeHalf];   // frame-axis cos/sin per staged frame
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
    int tiles_per_frame;           // ceil(T / kAttendKeys)
    int n_split;                   // key-range splits (grid z); 1: no partials
    int tiles_per_split;           // KV tiles per split (the last may hold fewer)
    float* part_o;                 // [n_split][M][H][D] unnormalised O per split
    float* part_ml;                // [n_split][M][H][2] (reference exponent, row sum)
    int debug_wait_fault;          // 1: producer never arms the first barrier
    long long wait_limit;          // per-wait limit in clock cycles
    int slot[kMaxSlots];           // key set, logical order
};

// Launchers (defined in the .cu files).
cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t stream);
cudaError_t launch_attend(const AttendParams& p, const CUtensorMap* maps, int D,
                          cudaStream_t stream);
// maps: [0] Q codes, [1] K codes, [2] V codes, [3] K scales, [4] V scales

}  // namespace rtv
