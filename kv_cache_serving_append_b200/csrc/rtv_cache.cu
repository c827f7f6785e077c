// rtv_cache.cu -- host side of librtv: configuration checks, device-buffer
// layout, ring bookkeeping, TMA descriptors and kernel launches behind the
// C ABI declared in include/rtv.h.
//
// Ring (aidose.in, "Runway explains how it serves a 57B video model in real
// time", third paragraph: the cache is a ring buffer that advances without
// copying; pttl.gr, section "Από οκτώ H100 σε τέσσερις": circular buffer):
// P0 pinned slots, then C = W + F_max ring slots.  Generated frame g lives in
// slot P0 + (g mod C); advancing moves the head and the visible window and
// touches no device memory.  Attention addresses frames through their slots
// inside the TMA coordinates, so a frame is written once and never moved.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <mutex>
#include <vector>

#include "rtv_internal.h"

using namespace rtv;

struct rtv_cache {
    rtv_cache_config cfg;
    int device = 0;
    int T = 0, S = 0, C = 0, P0 = 0, F_max = 0, W = 0, H = 0, D = 0;
    size_t bytes = 0;
    uint8_t* buf = nullptr;
    bool owns = false;
    std::vector<rtv_layer_layout> layout;
    float* h_table = nullptr;
    float* w_table = nullptr;
    unsigned int* err = nullptr;
    DeviceRing* dring = nullptr;        // ring state read by the kernels of a step graph
    float* part_o = nullptr;            // key-range split partials of one attention call
    int sm_count = 148;
    int last_splits = 0;
    // ring state
    long long G = 0;
    bool pinned_committed = false;
    std::vector<int> staged;            // frames staged per layer (0 = none)
    std::vector<long long> frame_of_slot;
    std::vector<long long> visible_frames;   // logical order
    std::vector<int> visible_slots;
    unsigned int seq = 0;
    std::vector<CUtensorMap> maps;      // 5 per layer: Q, K, V, K scales, V scales
    int debug_wait_fault = 0;
    int debug_bad_slot = -1;            // debug builds: slot the next attention names first
    long long wait_limit = 2000000000LL;
};

namespace {

constexpr size_t kAlign = 1024;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int round_up_int(int x, int a) { return (x + a - 1) / a * a; }

rtv_status validate(const rtv_cache_config* c)
{
    if (!c) return RTV_ERR_INVALID_ARG;
    if (c->n_layers < 1 || c->n_heads < 1 || c->grid_h < 1 || c->grid_w < 1 ||
        c->max_frames_per_chunk < 1 || c->window_frames < 0 || c->pinned_frames < 0 ||
        c->pinned_frames > 1 || c->rope_t < 0 || c->rope_h < 0 || c->rope_w < 0 ||
        !(c->rope_base > 0.0))
        return RTV_ERR_INVALID_ARG;
    if (c->rope_t + c->rope_h + c->rope_w != c->head_dim) return RTV_ERR_INVALID_ARG;
    if ((c->rope_t | c->rope_h | c->rope_w) & 1) return RTV_ERR_INVALID_ARG;
    if (c->head_dim != 64 && c->head_dim != 128) return RTV_ERR_UNSUPPORTED;
    if (c->n_heads > kMaxHeads) return RTV_ERR_UNSUPPORTED;
    if (c->max_frames_per_chunk > kMaxFrames) return RTV_ERR_UNSUPPORTED;
    const int E = c->head_dim / 16;
    if ((c->rope_t / 2) % E || (c->rope_h / 2) % E || (c->rope_w / 2) % E) return RTV_ERR_UNSUPPORTED;
    if (c->rope_t / 2 > kMaxRopeHalf) return RTV_ERR_UNSUPPORTED;
    const long long slots = (long long)c->pinned_frames + c->window_frames + c->max_frames_per_chunk;
    if (slots > kMaxSlots) return RTV_ERR_UNSUPPORTED;
    const long long T = (long long)c->grid_h * c->grid_w;
    if (T * c->max_frames_per_chunk > (1LL << 30) || slots * c->n_heads > (1LL << 30))
        return RTV_ERR_UNSUPPORTED;
    return RTV_OK;
}

struct Geometry {
    int T, S, q_rows, scale_pitch, q_scale_pitch;
    size_t layer_bytes, tables_off, split_off, err_off, ring_off, total;
    rtv_layer_layout rel;   // offsets relative to the layer base
};

Geometry geometry(const rtv_cache_config* c)
{
    Geometry g{};
    g.T = c->grid_h * c->grid_w;
    g.S = c->pinned_frames + c->window_frames + c->max_frames_per_chunk;
    g.q_rows = c->max_frames_per_chunk * g.T;
    g.scale_pitch = round_up_int(g.T, 16);
    g.q_scale_pitch = round_up_int(g.q_rows, 16);
    const size_t SH = (size_t)g.S * c->n_heads;
    size_t off = 0;
    g.rel.k_codes = off; off = align_up(off + SH * g.T * c->head_dim, kAlign);
    g.rel.v_codes = off; off = align_up(off + SH * g.T * c->head_dim, kAlign);
    g.rel.k_scales = off; off = align_up(off + SH * g.scale_pitch * 4, kAlign);
    g.rel.v_scales = off; off = align_up(off + SH * g.scale_pitch * 4, kAlign);
    g.rel.q_codes = off; off = align_up(off + (size_t)c->n_heads * g.q_rows * c->head_dim, kAlign);
    g.rel.q_scales = off; off = align_up(off + (size_t)c->n_heads * g.q_scale_pitch * 4, kAlign);
    g.rel.v_scale_max = off; off = align_up(off + SH * 8, kAlign);
    g.rel.scale_pitch = g.scale_pitch;
    g.rel.q_scale_pitch = g.q_scale_pitch;
    g.layer_bytes = off;
    g.tables_off = g.layer_bytes * c->n_layers;
    const size_t table_bytes = ((size_t)c->grid_h * c->rope_h + (size_t)c->grid_w * c->rope_w) * 4;
    // partials of the key-range splits, room for kMaxSplit x q_rows x H rows of
    // D + 2 floats (O, then the statistics; shared by all layers: one call at a time)
    const size_t split_rows = (size_t)kMaxSplit * g.q_rows * c->n_heads;
    g.split_off = align_up(g.tables_off + table_bytes, kAlign);
    g.err_off = align_up(g.split_off + split_rows * (c->head_dim + 2) * 4, kAlign);
    g.ring_off = align_up(g.err_off + 256, kAlign);
    g.total = align_up(g.ring_off + sizeof(DeviceRing), kAlign);
    return g;
}

// cos/sin table of one RoPE axis: [n_pos][2][n/2], angle pos * base^(-2j/n) in fp64.
void axis_table(std::vector<float>& out, int n_pos, int n, double base)
{
    const int half = n / 2;
    out.assign((size_t)n_pos * 2 * half, 0.f);
    for (int pos = 0; pos < n_pos; ++pos)
        for (int j = 0; j < half; ++j) {
            const double inv_freq = std::pow(base, -2.0 * (double)j / (double)n);
            const double theta = (double)pos * inv_freq;
            out[(size_t)pos * 2 * half + j] = (float)std::cos(theta);
            out[(size_t)pos * 2 * half + half + j] = (float)std::sin(theta);
        }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, void* base, const cuuint64_t* dims,
            const cuuint64_t* strides_bytes, const cuuint32_t* box, CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, dt, (cuuint32_t)rank, base, dims, strides_bytes, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool build_maps(rtv_cache* c)
{
    c->maps.resize((size_t)c->cfg.n_layers * 5);
    const int D = c->D, H = c->H, T = c->T, S = c->S;
    const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    for (int l = 0; l < c->cfg.n_layers; ++l) {
        const rtv_layer_layout& L = c->layout[l];
        CUtensorMap* m = &c->maps[(size_t)l * 5];
        const int q_rows = c->F_max * T;
        {   // Q codes [H][q_rows][D]
            cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)q_rows, (cuuint64_t)H};
            cuuint64_t st[2] = {(cuuint64_t)D, (cuuint64_t)q_rows * D};
            cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)kAttendRows, 1};
            if (!encode(&m[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, c->buf + L.q_codes, dims, st, box, sw))
                return false;
        }
        for (int kv = 0; kv < 2; ++kv) {   // K/V codes [S*H][T][D]
            cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)S * H};
            cuuint64_t st[2] = {(cuuint64_t)D, (cuuint64_t)T * D};
            cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)kAttendKeys, 1};
            if (!encode(&m[1 + kv], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                        c->buf + (kv ? L.v_codes : L.k_codes), dims, st, box, sw))
                return false;
        }
        for (int kv = 0; kv < 2; ++kv) {   // scales [S*H][scale_pitch] (first T used)
            cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)S * H};
            cuuint64_t st[1] = {(cuuint64_t)L.scale_pitch * 4};
            cuuint32_t box[2] = {(cuuint32_t)kAttendKeys, 1};
            if (!encode(&m[3 + kv], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                        c->buf + (kv ? L.v_scales : L.k_scales), dims, st, box,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
                return false;
        }
    }
    return true;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

bool same_device(const rtv_cache* c)
{
    int d = -1;
    return cudaGetDevice(&d) == cudaSuccess && d == c->device;
}

int frames_committed(const rtv_cache* c) { return (c->pinned_committed ? 1 : 0) + (int)c->G; }

bool in_pinned_phase(const rtv_cache* c) { return c->P0 == 1 && !c->pinned_committed; }

int staged_slot(const rtv_cache* c, int f)
{
    if (in_pinned_phase(c)) return 0;
    return c->P0 + (int)((c->G + f) % c->C);
}

// Frame-axis RoPE cos/sin of absolute frame t: angle t * base^(-2j/rope_t) in fp64.
void frame_table(const rtv_cache* c, long long t, float (*tt)[kMaxRopeHalf])
{
    const int half = c->cfg.rope_t / 2;
    for (int j = 0; j < half; ++j) {
        const double inv_freq = std::pow(c->cfg.rope_base, -2.0 * (double)j / (double)c->cfg.rope_t);
        const double theta = (double)t * inv_freq;
        tt[0][j] = (float)std::cos(theta);
        tt[1][j] = (float)std::sin(theta);
    }
}

// Launch parameters of one layer's append (no change to the cache's state).
void fill_append_params(const rtv_cache* c, int layer, const void* q, const void* k, const void* v,
                        int n_frames, unsigned int seq, AppendParams& p)
{
    const rtv_layer_layout& L = c->layout[layer];
    std::memset(&p, 0, sizeof p);
    p.neg_zero = -0.0f;
    p.one = 1.0f;
    p.src[0] = static_cast<const uint16_t*>(q);
    p.src[1] = static_cast<const uint16_t*>(k);
    p.src[2] = static_cast<const uint16_t*>(v);
    p.q_codes = c->buf + L.q_codes;
    p.q_scales = reinterpret_cast<float*>(c->buf + L.q_scales);
    p.kv_codes[0] = c->buf + L.k_codes;
    p.kv_codes[1] = c->buf + L.v_codes;
    p.kv_scales[0] = reinterpret_cast<float*>(c->buf + L.k_scales);
    p.kv_scales[1] = reinterpret_cast<float*>(c->buf + L.v_scales);
    p.v_scale_max = reinterpret_cast<unsigned long long*>(c->buf + L.v_scale_max);
    p.h_table = c->h_table;
    p.w_table = c->w_table;
    p.H = c->H; p.D = c->D; p.T = c->T; p.grid_w = c->cfg.grid_w; p.n_frames = n_frames;
    p.q_rows = c->F_max * c->T;
    p.q_scale_pitch = L.q_scale_pitch;
    p.scale_pitch = L.scale_pitch;
    p.n_t = c->cfg.rope_t; p.n_h = c->cfg.rope_h; p.n_w = c->cfg.rope_w;
    p.seq = seq;
    p.n_slots = c->S;
    p.err = c->err;
    const long long t0 = frames_committed(c);
    for (int f = 0; f < n_frames; ++f) {
        p.slot[f] = staged_slot(c, f);
        frame_table(c, t0 + f, p.t_table[f]);
    }
}

// Launch parameters of one layer's attention over n staged frames (no change
// to the cache's state).  The split partials go to part_base (capacity_bytes
// of room: n_split*M*H*D floats of O, then n_split*M*H*2 of statistics); a
// plan whose partials do not fit is rejected with RTV_ERR_UNSUPPORTED.
rtv_status fill_attend_params(const rtv_cache* c, int layer, void* out, int out_dtype, int n,
                              float* part_base, size_t capacity_bytes, AttendParams& p)
{
    const rtv_layer_layout& L = c->layout[layer];
    std::memset(&p, 0, sizeof p);
    p.q_scales = reinterpret_cast<const float*>(c->buf + L.q_scales);
    p.v_scale_max = reinterpret_cast<const unsigned long long*>(c->buf + L.v_scale_max);
    p.out = out;
    p.err = c->err;
    p.H = c->H; p.D = c->D; p.T = c->T; p.M = n * c->T;
    p.q_scale_pitch = L.q_scale_pitch;
    p.out_bf16 = out_dtype == RTV_OUT_BF16;
    p.key_tile = kAttendKeys;
    p.tiles_per_frame = (c->T + kAttendKeys - 1) / kAttendKeys;
    int nk = 0;
    for (int s : c->visible_slots) p.slot[nk++] = s;
    for (int f = 0; f < n; ++f) p.slot[nk++] = staged_slot(c, f);
    p.n_frames_keys = nk;
    const int units = ((p.M + 2 * kAttendRows - 1) / (2 * kAttendRows)) * p.H;
    if (rtv_split_plan(units, nk * p.tiles_per_frame, c->sm_count, &p.n_split, &p.tiles_per_split) != RTV_OK)
        return RTV_ERR_INVALID_ARG;
    const size_t part_rows = (size_t)p.n_split * p.M * p.H;
    if (p.n_split > 1 && part_rows * (p.D + 2) * sizeof(float) > capacity_bytes) return RTV_ERR_UNSUPPORTED;
    p.part_o = part_base;
    p.part_ml = part_base + part_rows * p.D;
    p.n_slots = c->S;
    p.debug_wait_fault = c->debug_wait_fault;
    p.wait_limit = c->wait_limit;
    return RTV_OK;
}

// Commit n staged frames to the host ring state (no device work).
void commit_frames(rtv_cache* c, int n)
{
    const long long t0 = frames_committed(c);
    for (int f = 0; f < n; ++f) {
        const int s = staged_slot(c, f);
        c->frame_of_slot[s] = t0 + f;
        c->visible_frames.push_back(t0 + f);
        c->visible_slots.push_back(s);
    }
    if (in_pinned_phase(c)) c->pinned_committed = true;
    else c->G += n;
    const size_t n_pinned = c->pinned_committed ? 1 : 0;
    while (c->visible_frames.size() - n_pinned > (size_t)c->W) {
        c->frame_of_slot[c->visible_slots[n_pinned]] = -1;
        c->visible_frames.erase(c->visible_frames.begin() + n_pinned);
        c->visible_slots.erase(c->visible_slots.begin() + n_pinned);
    }
    std::fill(c->staged.begin(), c->staged.end(), 0);
}

// The steady state a step graph can capture: pinned frame committed, window
// full, nothing staged.
bool steady(const rtv_cache* c)
{
    if (c->P0 && !c->pinned_committed) return false;
    if (c->G < c->W) return false;
    for (int n : c->staged)
        if (n) return false;
    return true;
}

// The device ring state of the current host state for chunks of n frames.
void host_ring(const rtv_cache* c, int n, DeviceRing& r)
{
    std::memset(&r, 0, sizeof r);
    r.G = c->G;
    r.t0 = frames_committed(c);
    r.seq = c->seq + 1;
    int nk = 0;
    for (int s : c->visible_slots) r.slot[nk++] = s;
    for (int f = 0; f < n; ++f) {
        r.staged_slot[f] = staged_slot(c, f);
        r.slot[nk++] = r.staged_slot[f];
        frame_table(c, r.t0 + f, r.t_table[f]);
    }
    r.n_staged = n;
    r.P0 = c->P0;
    r.C = c->C;
    r.W = c->W;
    r.n_keys = nk;
    r.rope_half = c->cfg.rope_t / 2;
    for (int j = 0; j < r.rope_half; ++j)
        r.inv_freq[j] = std::pow(c->cfg.rope_base, -2.0 * (double)j / (double)c->cfg.rope_t);
}

// Advance of the device ring state by one chunk (steady state): one warp.
// The window is generated frames G-W..G-1, the staged frames G..G+F-1, every
// one in slot P0 + (g mod C); the frame-axis cos/sin of the new staged frames
// use the host's fp64 inverse frequencies and the device's fp64 sincos.
__global__ void ring_advance_kernel(DeviceRing* r)
{
    const int lane = threadIdx.x;
    const int F = r->n_staged, P0 = r->P0, C = r->C, W = r->W;
    const long long G = r->G + F;
    const long long t0 = r->t0 + F;
    const unsigned int seq = r->seq + 1;
    __syncwarp();
    for (int i = lane; i < r->n_keys; i += 32)
        r->slot[i] = i < P0 ? 0 : P0 + (int)((G - W + (i - P0)) % C);
    for (int f = lane; f < F; f += 32) r->staged_slot[f] = P0 + (int)((G + f) % C);
    for (int i = lane; i < F * r->rope_half; i += 32) {
        const int f = i / r->rope_half, j = i - f * r->rope_half;
        double sn, cs;
        sincos((double)(t0 + f) * r->inv_freq[j], &sn, &cs);
        r->t_table[f][0][j] = (float)cs;
        r->t_table[f][1][j] = (float)sn;
    }
    __syncwarp();
    if (lane == 0) {
        r->G = G;
        r->t0 = t0;
        r->seq = seq;
    }
}

// Split partials of rtv_attend_static_scratch: a fixed device array (16 MiB),
// shared by every cache and stream of the device.
constexpr size_t kStaticScratchFloats = (size_t)4 << 20;
__device__ __align__(256) float g_static_scratch[kStaticScratchFloats];

// Address of g_static_scratch on the current device, looked up once per device.
rtv_status static_scratch_address(int device, float** out)
{
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    if (device < 0 || device >= kMaxDevices) return RTV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[device]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_static_scratch) != cudaSuccess || !a) {
            cudaGetLastError();
            return RTV_ERR_CUDA;
        }
        addr[device] = a;
    }
    *out = static_cast<float*>(addr[device]);
    return RTV_OK;
}

}  // namespace

namespace rtv {
cudaError_t launch_ring_advance(DeviceRing* ring, cudaStream_t stream)
{
    ring_advance_kernel<<<1, 32, 0, stream>>>(ring);
    return cudaGetLastError();
}
}  // namespace rtv

struct rtv_step_graph {
    rtv_cache* cache = nullptr;
    int n_frames = 0;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    long long valid_G = -1;             // host state for which the device ring is current
    unsigned int valid_seq = 0;
};

extern "C" {

const char* rtv_status_string(rtv_status s)
{
    switch (s) {
    case RTV_OK: return "ok";
    case RTV_ERR_INVALID_ARG: return "invalid argument";
    case RTV_ERR_OOM: return "out of device memory";
    case RTV_ERR_CUDA: return "CUDA error";
    case RTV_ERR_STATE: return "invalid state for this call";
    case RTV_ERR_TIMEOUT: return "kernel wait timed out";
    case RTV_ERR_UNSUPPORTED: return "unsupported configuration";
    case RTV_ERR_BOUNDS: return "slot index out of range (debug build)";
    }
    return "unknown status";
}

rtv_status rtv_cache_required_bytes(const rtv_cache_config* cfg, size_t* bytes)
{
    if (!bytes) return RTV_ERR_INVALID_ARG;
    rtv_status st = validate(cfg);
    if (st != RTV_OK) return st;
    *bytes = geometry(cfg).total;
    return RTV_OK;
}

rtv_status rtv_cache_layer_layout(const rtv_cache_config* cfg, int layer, rtv_layer_layout* out)
{
    if (!out) return RTV_ERR_INVALID_ARG;
    rtv_status st = validate(cfg);
    if (st != RTV_OK) return st;
    if (layer < 0 || layer >= cfg->n_layers) return RTV_ERR_INVALID_ARG;
    Geometry g = geometry(cfg);
    rtv_layer_layout L = g.rel;
    const size_t base = g.layer_bytes * layer;
    L.k_codes += base; L.v_codes += base; L.k_scales += base; L.v_scales += base;
    L.q_codes += base; L.q_scales += base; L.v_scale_max += base;
    *out = L;
    return RTV_OK;
}

rtv_status rtv_cache_create(const rtv_cache_config* cfg, void* device_buf, size_t buf_bytes,
                            rtv_cache** out)
{
    if (!out) return RTV_ERR_INVALID_ARG;
    *out = nullptr;
    rtv_status st = validate(cfg);
    if (st != RTV_OK) return st;
    Geometry g = geometry(cfg);
    if (device_buf && (buf_bytes < g.total || ((uintptr_t)device_buf & 255))) return RTV_ERR_INVALID_ARG;

    if (!device_buf) {
        // host-side fault injection for the out-of-memory path (tests)
        const char* inj = std::getenv("RTV_INJECT_ALLOC_FAILURE");
        if (inj && inj[0] == '1') return RTV_ERR_OOM;
    }
    rtv_cache* c = new (std::nothrow) rtv_cache();
    if (!c) return RTV_ERR_OOM;
    c->cfg = *cfg;
    if (cudaGetDevice(&c->device) != cudaSuccess) { delete c; return RTV_ERR_CUDA; }
    c->T = g.T; c->S = g.S; c->P0 = cfg->pinned_frames; c->F_max = cfg->max_frames_per_chunk;
    c->W = cfg->window_frames; c->C = c->W + c->F_max; c->H = cfg->n_heads; c->D = cfg->head_dim;
    c->bytes = g.total;
    if (device_buf) {
        c->buf = static_cast<uint8_t*>(device_buf);
    } else {
        if (cudaMalloc(&c->buf, g.total) != cudaSuccess) {
            cudaGetLastError();
            delete c;
            return RTV_ERR_OOM;
        }
        c->owns = true;
    }
    for (int l = 0; l < cfg->n_layers; ++l) {
        rtv_layer_layout L;
        rtv_cache_layer_layout(cfg, l, &L);
        c->layout.push_back(L);
    }
    c->h_table = reinterpret_cast<float*>(c->buf + g.tables_off);
    c->w_table = c->h_table + (size_t)cfg->grid_h * cfg->rope_h;
    c->err = reinterpret_cast<unsigned int*>(c->buf + g.err_off);
    c->dring = reinterpret_cast<DeviceRing*>(c->buf + g.ring_off);
    c->part_o = reinterpret_cast<float*>(c->buf + g.split_off);
    {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c->device) == cudaSuccess && sms > 0)
            c->sm_count = sms;
        else
            cudaGetLastError();
    }
    c->staged.assign(cfg->n_layers, 0);
    c->frame_of_slot.assign(c->S, -1);

    std::vector<float> ht, wt;
    axis_table(ht, cfg->grid_h, cfg->rope_h, cfg->rope_base);
    axis_table(wt, cfg->grid_w, cfg->rope_w, cfg->rope_base);
    bool ok = cudaMemset(c->buf, 0, g.total) == cudaSuccess;
    if (ok && !ht.empty())
        ok = cudaMemcpy(c->h_table, ht.data(), ht.size() * 4, cudaMemcpyHostToDevice) == cudaSuccess;
    if (ok && !wt.empty())
        ok = cudaMemcpy(c->w_table, wt.data(), wt.size() * 4, cudaMemcpyHostToDevice) == cudaSuccess;
    if (ok) ok = cudaDeviceSynchronize() == cudaSuccess;
    if (ok) {
        // Resolve the allocation-free entry point's device array now, so the
        // module that holds it is loaded at set-up (under lazy module loading
        // its 16 MiB are reserved here, not by a later attention call).  A
        // failure is not fatal to the cache: rtv_attend_static_scratch then
        // retries and reports it.
        float* scratch = nullptr;
        if (static_scratch_address(c->device, &scratch) != RTV_OK) cudaGetLastError();
    }
    if (ok && !build_maps(c)) {
        if (c->owns) cudaFree(c->buf);
        delete c;
        return RTV_ERR_CUDA;
    }
    if (!ok) {
        cudaGetLastError();
        if (c->owns) cudaFree(c->buf);
        delete c;
        return RTV_ERR_CUDA;
    }
    *out = c;
    return RTV_OK;
}

rtv_status rtv_cache_destroy(rtv_cache* c)
{
    if (!c) return RTV_ERR_INVALID_ARG;
    rtv_status st = RTV_OK;
    if (cudaDeviceSynchronize() != cudaSuccess) st = RTV_ERR_CUDA;
    if (c->owns && cudaFree(c->buf) != cudaSuccess) st = RTV_ERR_CUDA;
    delete c;
    return st;
}

rtv_status rtv_cache_append(rtv_cache* c, int layer, const void* q, const void* k, const void* v,
                            int n_frames, void* stream)
{
    if (!c || layer < 0 || layer >= c->cfg.n_layers) return RTV_ERR_INVALID_ARG;
    if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return RTV_ERR_INVALID_ARG;
    if (n_frames < 1 || n_frames > c->F_max) return RTV_ERR_INVALID_ARG;
    if (in_pinned_phase(c) && n_frames != 1) return RTV_ERR_INVALID_ARG;
    for (int l = 0; l < c->cfg.n_layers; ++l)
        if (l != layer && c->staged[l] && c->staged[l] != n_frames) return RTV_ERR_STATE;
    if (!same_device(c)) return RTV_ERR_INVALID_ARG;

    AppendParams p;
    fill_append_params(c, layer, q, k, v, n_frames, ++c->seq, p);
    if (launch_append(p, c->D, static_cast<cudaStream_t>(stream)) != cudaSuccess) return RTV_ERR_CUDA;
    c->staged[layer] = n_frames;
    return RTV_OK;
}

rtv_status rtv_cache_append_project(rtv_cache* c, int layer, const void* x_codes, const float* x_scales,
                                    const void* w_codes, const float* w_scales, int hidden, int n_frames,
                                    void* stream)
{
    if (!c || layer < 0 || layer >= c->cfg.n_layers) return RTV_ERR_INVALID_ARG;
    if (!x_codes || !x_scales || !w_codes || !w_scales || !aligned16(x_codes) || !aligned16(w_codes) ||
        !aligned16(w_scales) || ((uintptr_t)x_scales & 3))
        return RTV_ERR_INVALID_ARG;
    if (hidden < 128 || hidden % 128) return RTV_ERR_INVALID_ARG;
    if (n_frames < 1 || n_frames > c->F_max) return RTV_ERR_INVALID_ARG;
    if (in_pinned_phase(c) && n_frames != 1) return RTV_ERR_INVALID_ARG;
    // the fused epilogue is specialised to the workloads' head shape
    if (c->D != 128 || c->cfg.rope_t != 32 || c->cfg.rope_h != 48 || c->cfg.rope_w != 48 || (c->H % 2))
        return RTV_ERR_UNSUPPORTED;
    for (int l = 0; l < c->cfg.n_layers; ++l)
        if (l != layer && c->staged[l] && c->staged[l] != n_frames) return RTV_ERR_STATE;
    if (!same_device(c)) return RTV_ERR_INVALID_ARG;
    const int rows = n_frames * c->T;
    const int feats = 3 * c->H * c->D;
    CUtensorMap maps[2];
    {
        cuuint64_t dims[2] = {(cuuint64_t)hidden, (cuuint64_t)rows};
        cuuint64_t st[1] = {(cuuint64_t)hidden};
        cuuint32_t box[2] = {128, 128};
        if (!encode(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(x_codes), dims, st, box,
                    CU_TENSOR_MAP_SWIZZLE_128B))
            return RTV_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)hidden, (cuuint64_t)feats};
        cuuint64_t st[1] = {(cuuint64_t)hidden};
        cuuint32_t box[2] = {128, 256};
        if (!encode(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(w_codes), dims, st, box,
                    CU_TENSOR_MAP_SWIZZLE_128B))
            return RTV_ERR_CUDA;
    }
    ProjectParams p;
    std::memset(&p, 0, sizeof p);
    fill_append_params(c, layer, nullptr, nullptr, nullptr, n_frames, ++c->seq, p.a);
    p.sx = x_scales;
    p.sw = w_scales;
    p.R = rows;
    p.Kd = hidden;
    p.n_m_tiles = (rows + 127) / 128;
    p.n_n_tiles = feats / 256;
    p.wait_limit = c->wait_limit;
    p.err = c->err;
    if (launch_project(p, maps, c->sm_count, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return RTV_ERR_CUDA;
    }
    c->staged[layer] = n_frames;
    return RTV_OK;
}

rtv_status rtv_split_plan(int n_units, int n_kv_tiles, int sm_count, int* n_split, int* tiles_per_split)
{
    if (n_units < 1 || n_kv_tiles < 1 || sm_count < 1 || !n_split || !tiles_per_split)
        return RTV_ERR_INVALID_ARG;
    // One CTA per unit alone gives ceil(units / SMs) waves of equal CTAs;
    // splitting every unit's key range s ways fills the last wave better at
    // the price of a merge pass.  Pick s with the least ceil(units * s / SMs)
    // / s, charging 3% of a full-range CTA per extra split (pipeline fill and
    // drain, partial write and merge), and keep at least 8 KV tiles per split.
    int best_s = 1;
    double best_cost = 1e30;
    for (int s = 1; s <= kMaxSplit; ++s) {
        if (s > 1 && n_kv_tiles / s < 8) break;
        const long long waves = ((long long)n_units * s + sm_count - 1) / sm_count;
        const double cost = (double)waves / s + 0.03 * (s - 1);
        if (cost < best_cost - 1e-9) { best_cost = cost; best_s = s; }
    }
    const int tps = (n_kv_tiles + best_s - 1) / best_s;
    *tiles_per_split = tps;
    *n_split = (n_kv_tiles + tps - 1) / tps;   // no empty split
    return RTV_OK;
}

namespace {

// Attention launch shared by rtv_attend and rtv_attend_static_scratch.  The
// split partials go to part_o / part_ml (capacity_bytes of room, in floats:
// n_split*M*H*D of O, then n_split*M*H*2 of statistics); a plan whose
// partials do not fit is rejected with RTV_ERR_UNSUPPORTED before any launch.
rtv_status attend_impl(rtv_cache* c, int layer, void* out, int out_dtype, void* stream,
                       float* part_base, size_t capacity_bytes)
{
    if (!c || layer < 0 || layer >= c->cfg.n_layers) return RTV_ERR_INVALID_ARG;
    if (!out || !aligned16(out)) return RTV_ERR_INVALID_ARG;
    if (out_dtype != RTV_OUT_F32 && out_dtype != RTV_OUT_BF16) return RTV_ERR_INVALID_ARG;
    const int n = c->staged[layer];
    if (n == 0) return RTV_ERR_STATE;
    if (!same_device(c)) return RTV_ERR_INVALID_ARG;

    AttendParams p;
    const rtv_status st = fill_attend_params(c, layer, out, out_dtype, n, part_base, capacity_bytes, p);
    if (st != RTV_OK) return st;
    c->debug_wait_fault = 0;
    if (c->debug_bad_slot >= 0) {
        p.slot[0] = c->debug_bad_slot;   // only reachable in a debug build
        c->debug_bad_slot = -1;
    }
    c->last_splits = p.n_split;
    if (launch_attend(p, &c->maps[(size_t)layer * 5], c->D, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return RTV_ERR_CUDA;
    return RTV_OK;
}

}  // namespace

rtv_status rtv_attend(rtv_cache* c, int layer, void* out, int out_dtype, void* stream)
{
    if (!c) return RTV_ERR_INVALID_ARG;
    // the cache buffer's split section holds kMaxSplit * F_max*T * H rows
    const size_t cap = (size_t)kMaxSplit * c->F_max * c->T * c->H * (c->D + 2) * sizeof(float);
    return attend_impl(c, layer, out, out_dtype, stream, c->part_o, cap);
}

rtv_status rtv_attend_static_scratch(rtv_cache* c, int layer, void* out, int out_dtype, void* stream)
{
    if (!c) return RTV_ERR_INVALID_ARG;
    if (!same_device(c)) return RTV_ERR_INVALID_ARG;
    float* base = nullptr;
    const rtv_status st = static_scratch_address(c->device, &base);
    if (st != RTV_OK) return st;
    return attend_impl(c, layer, out, out_dtype, stream, base, kStaticScratchFloats * sizeof(float));
}

rtv_status rtv_cache_advance(rtv_cache* c)
{
    if (!c) return RTV_ERR_INVALID_ARG;
    const int n = c->staged[0];
    if (n == 0) return RTV_ERR_STATE;
    for (int l = 1; l < c->cfg.n_layers; ++l)
        if (c->staged[l] != n) return RTV_ERR_STATE;
    for (int f = 0; f < n; ++f) {
        const int s = staged_slot(c, f);
        if (c->frame_of_slot[s] != -1) return RTV_ERR_STATE;   // cannot happen: F <= F_max
    }
    commit_frames(c, n);
    return RTV_OK;
}

rtv_status rtv_cache_get_state(const rtv_cache* c, rtv_cache_state* out)
{
    if (!c || !out) return RTV_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof *out);
    out->frames_committed = frames_committed(c);
    out->generated_committed = c->G;
    out->pinned_committed = c->pinned_committed ? 1 : 0;
    out->head = c->P0 + (int)(c->G % c->C);
    out->n_slots = c->S;
    out->n_visible = (int)c->visible_frames.size();
    for (int i = 0; i < out->n_visible; ++i) {
        out->visible_frames[i] = c->visible_frames[i];
        out->visible_slots[i] = c->visible_slots[i];
    }
    for (int s = 0; s < RTV_MAX_SLOTS; ++s) out->frame_of_slot[s] = s < c->S ? c->frame_of_slot[s] : -1;
    int ns = 0, nf = 0;
    for (int l = 0; l < c->cfg.n_layers; ++l)
        if (c->staged[l]) {
            if (ns == 0) nf = c->staged[l];
            else if (nf != c->staged[l]) nf = -1;
            ++ns;
        }
    out->staged_layers = ns;
    out->staged_frames = nf;
    out->last_attend_splits = c->last_splits;
    return RTV_OK;
}

rtv_status rtv_cache_device_buffer(const rtv_cache* c, void** ptr, size_t* bytes)
{
    if (!c || !ptr || !bytes) return RTV_ERR_INVALID_ARG;
    *ptr = c->buf;
    *bytes = c->bytes;
    return RTV_OK;
}

rtv_status rtv_cache_export(const rtv_cache* c, int layer, int slot, void* codes_k, void* codes_v,
                            float* sk, float* sv, void* q_codes, float* sq, void* stream)
{
    if (!c || layer < 0 || layer >= c->cfg.n_layers || slot < 0 || slot >= c->S)
        return RTV_ERR_INVALID_ARG;
    const rtv_layer_layout& L = c->layout[layer];
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t plane = (size_t)c->H * c->T * c->D;
    bool ok = true;
    if (codes_k) ok &= cudaMemcpyAsync(codes_k, c->buf + L.k_codes + plane * slot, plane, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    if (codes_v) ok &= cudaMemcpyAsync(codes_v, c->buf + L.v_codes + plane * slot, plane, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    const size_t pitch = (size_t)L.scale_pitch * 4;
    const size_t sbase = (size_t)slot * c->H * pitch;
    if (sk) ok &= cudaMemcpy2DAsync(sk, (size_t)c->T * 4, c->buf + L.k_scales + sbase, pitch, (size_t)c->T * 4, c->H, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    if (sv) ok &= cudaMemcpy2DAsync(sv, (size_t)c->T * 4, c->buf + L.v_scales + sbase, pitch, (size_t)c->T * 4, c->H, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    const size_t q_rows = (size_t)c->F_max * c->T;
    if (q_codes) ok &= cudaMemcpyAsync(q_codes, c->buf + L.q_codes, (size_t)c->H * q_rows * c->D, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    if (sq) ok &= cudaMemcpy2DAsync(sq, q_rows * 4, c->buf + L.q_scales, (size_t)L.q_scale_pitch * 4, q_rows * 4, c->H, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    if (ok) ok = cudaStreamSynchronize(s) == cudaSuccess;
    if (!ok) cudaGetLastError();
    return ok ? RTV_OK : RTV_ERR_CUDA;
}

rtv_status rtv_poll_error(rtv_cache* c)
{
    if (!c) return RTV_ERR_INVALID_ARG;
    unsigned int e = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return RTV_ERR_CUDA;
    if (cudaMemcpy(&e, c->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return RTV_ERR_CUDA;
    if (e && cudaMemset(c->err, 0, 4) != cudaSuccess) return RTV_ERR_CUDA;
    if (e & kErrBounds) return RTV_ERR_BOUNDS;
    if (e & kErrTimeout) return RTV_ERR_TIMEOUT;
    return RTV_OK;
}

rtv_status rtv_debug_set_wait_fault(rtv_cache* c, int enable, long long wait_limit_cycles)
{
    if (!c || wait_limit_cycles < 0) return RTV_ERR_INVALID_ARG;
    c->debug_wait_fault = enable ? 1 : 0;
    c->wait_limit = wait_limit_cycles ? wait_limit_cycles : 2000000000LL;
    return RTV_OK;
}

int rtv_debug_build(void)
{
#ifdef RTV_DEBUG
    return 1;
#else
    return 0;
#endif
}

rtv_status rtv_debug_corrupt_next_attend(rtv_cache* c, int bad_slot)
{
    if (!c) return RTV_ERR_INVALID_ARG;
#ifdef RTV_DEBUG
    c->debug_bad_slot = bad_slot < 0 ? -1 : bad_slot;
    return RTV_OK;
#else
    (void)bad_slot;
    return RTV_ERR_UNSUPPORTED;
#endif
}

rtv_status rtv_step_graph_create(rtv_cache* c, int n_frames, const void* const* q,
                                 const void* const* k, const void* const* v, void* const* out,
                                 int out_dtype, void* stream, rtv_step_graph** out_graph)
{
    if (!out_graph) return RTV_ERR_INVALID_ARG;
    *out_graph = nullptr;
    if (!c || !q || !k || !v || !out || !stream) return RTV_ERR_INVALID_ARG;
    if (n_frames < 1 || n_frames > c->F_max) return RTV_ERR_INVALID_ARG;
    if (out_dtype != RTV_OUT_F32 && out_dtype != RTV_OUT_BF16) return RTV_ERR_INVALID_ARG;
    const int L = c->cfg.n_layers;
    for (int l = 0; l < L; ++l)
        if (!q[l] || !k[l] || !v[l] || !out[l] || !aligned16(q[l]) || !aligned16(k[l]) ||
            !aligned16(v[l]) || !aligned16(out[l]))
            return RTV_ERR_INVALID_ARG;
    if (!same_device(c)) return RTV_ERR_INVALID_ARG;
    if (!steady(c)) return RTV_ERR_STATE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (prepare_append(c->D) != cudaSuccess || prepare_attend(c->D) != cudaSuccess) {
        cudaGetLastError();
        return RTV_ERR_CUDA;
    }
    DeviceRing r;
    host_ring(c, n_frames, r);
    std::vector<AppendParams> ap(L);
    std::vector<AttendParams> tp(L);
    const size_t cap = (size_t)kMaxSplit * c->F_max * c->T * c->H * (c->D + 2) * sizeof(float);
    for (int l = 0; l < L; ++l) {
        fill_append_params(c, l, q[l], k[l], v[l], n_frames, r.seq, ap[l]);
        ap[l].ring = c->dring;
        const rtv_status st = fill_attend_params(c, l, out[l], out_dtype, n_frames, c->part_o, cap, tp[l]);
        if (st != RTV_OK) return st;
        tp[l].ring = c->dring;
        tp[l].debug_wait_fault = 0;
    }
    if (cudaMemcpyAsync(c->dring, &r, sizeof r, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return RTV_ERR_CUDA;
    }
    cudaGraph_t graph = nullptr;
    if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        cudaGetLastError();
        return RTV_ERR_CUDA;
    }
    bool ok = true;
    for (int l = 0; l < L && ok; ++l)
        ok = launch_append(ap[l], c->D, s) == cudaSuccess &&
             launch_attend(tp[l], &c->maps[(size_t)l * 5], c->D, s) == cudaSuccess;
    ok = ok && launch_ring_advance(c->dring, s) == cudaSuccess;
    const cudaError_t e = cudaStreamEndCapture(s, &graph);
    cudaGraphExec_t exec = nullptr;
    if (ok && e == cudaSuccess && graph) ok = cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
    else ok = false;
    rtv_step_graph* g = ok ? new (std::nothrow) rtv_step_graph() : nullptr;
    if (!g) {
        if (exec) cudaGraphExecDestroy(exec);
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();
        return ok ? RTV_ERR_OOM : RTV_ERR_CUDA;
    }
    g->cache = c;
    g->n_frames = n_frames;
    g->graph = graph;
    g->exec = exec;
    g->valid_G = c->G;
    g->valid_seq = c->seq;
    c->last_splits = tp[0].n_split;
    *out_graph = g;
    return RTV_OK;
}

rtv_status rtv_step_graph_launch(rtv_step_graph* g, void* stream)
{
    if (!g || !g->cache) return RTV_ERR_INVALID_ARG;
    rtv_cache* c = g->cache;
    if (!same_device(c)) return RTV_ERR_INVALID_ARG;
    if (!steady(c)) return RTV_ERR_STATE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (c->G != g->valid_G || c->seq != g->valid_seq) {
        // direct calls moved the ring since the last replay: bring the device
        // ring state up to date first (stream-ordered)
        DeviceRing r;
        host_ring(c, g->n_frames, r);
        if (cudaMemcpyAsync(c->dring, &r, sizeof r, cudaMemcpyHostToDevice, s) != cudaSuccess) {
            cudaGetLastError();
            return RTV_ERR_CUDA;
        }
    }
    if (cudaGraphLaunch(g->exec, s) != cudaSuccess) {
        cudaGetLastError();
        return RTV_ERR_CUDA;
    }
    // the host mirror makes the same step: every layer appended under one
    // sequence number, then the chunk committed
    c->seq += 1;
    commit_frames(c, g->n_frames);
    g->valid_G = c->G;
    g->valid_seq = c->seq;
    return RTV_OK;
}

rtv_status rtv_step_graph_destroy(rtv_step_graph* g)
{
    if (!g) return RTV_ERR_INVALID_ARG;
    rtv_status st = RTV_OK;
    if (g->exec && cudaGraphExecDestroy(g->exec) != cudaSuccess) st = RTV_ERR_CUDA;
    if (g->graph && cudaGraphDestroy(g->graph) != cudaSuccess) st = RTV_ERR_CUDA;
    delete g;
    return st;
}

}  // extern "C"
