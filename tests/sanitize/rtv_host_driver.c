/*
 * Drives the host-only paths of librtv's C ABI (configuration checks,
 * buffer geometry, the attention split plan, status strings, NULL and bad
 * arguments, the injected allocation failure) for a build of the library's
 * host code with AddressSanitizer and UndefinedBehaviorSanitizer (test
 * infrastructure; run by tests/test_sanitizers_cpu.py).  No call here reaches
 * a CUDA device.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "../../include/rtv.h"

static rtv_cache_config cfg(int layers, int heads, int D, int gh, int gw, int F, int W, int P0)
{
    rtv_cache_config c;
    memset(&c, 0, sizeof c);
    c.n_layers = layers; c.n_heads = heads; c.head_dim = D; c.grid_h = gh; c.grid_w = gw;
    c.max_frames_per_chunk = F; c.window_frames = W; c.pinned_frames = P0;
    c.rope_t = D / 4; c.rope_h = 3 * D / 8; c.rope_w = 3 * D / 8; c.rope_base = 10000.0;
    return c;
}

int main(void)
{
    int s, l, n, t;
    size_t bytes;
    rtv_layer_layout L;
    rtv_cache_config good[5];
    good[0] = cfg(1, 2, 64, 8, 8, 1, 4, 0);
    good[1] = cfg(2, 8, 128, 22, 32, 1, 6, 0);
    good[2] = cfg(1, 40, 128, 44, 68, 1, 8, 0);
    good[3] = cfg(48, 40, 128, 44, 68, 1, 8, 0);
    good[4] = cfg(1, 40, 128, 44, 68, 2, 16, 1);
    for (s = 0; s < 7; ++s)
        if (!rtv_status_string((rtv_status)s)) return 1;
    (void)rtv_status_string((rtv_status)99);
    for (s = 0; s < 5; ++s) {
        if (rtv_cache_required_bytes(&good[s], &bytes) != RTV_OK || bytes == 0) return 2;
        for (l = 0; l < good[s].n_layers; ++l)
            if (rtv_cache_layer_layout(&good[s], l, &L) != RTV_OK || L.k_codes + L.v_codes == 0) return 3;
        if (rtv_cache_layer_layout(&good[s], good[s].n_layers, &L) != RTV_ERR_INVALID_ARG) return 4;
    }
    {   /* rejected configurations */
        rtv_cache_config b = good[1];
        b.head_dim = 96; b.rope_t = 32; b.rope_h = 32; b.rope_w = 32;
        if (rtv_cache_required_bytes(&b, &bytes) == RTV_OK) return 5;
        b = good[1]; b.rope_t = 31;
        if (rtv_cache_required_bytes(&b, &bytes) == RTV_OK) return 6;
        b = good[1]; b.window_frames = 70;
        if (rtv_cache_required_bytes(&b, &bytes) == RTV_OK) return 7;
        b = good[1]; b.n_heads = 0;
        if (rtv_cache_required_bytes(&b, &bytes) == RTV_OK) return 8;
        if (rtv_cache_required_bytes(NULL, &bytes) != RTV_ERR_INVALID_ARG) return 9;
        if (rtv_cache_required_bytes(&good[0], NULL) != RTV_ERR_INVALID_ARG) return 10;
    }
    for (s = 1; s <= 2000; s += 37)
        for (l = 1; l <= 1200; l += 29)
            if (rtv_split_plan(s, l, 148, &n, &t) != RTV_OK || n < 1 || n > 4 || (n - 1) * t >= l || n * t < l)
                return 11;
    if (rtv_split_plan(0, 1, 148, &n, &t) != RTV_ERR_INVALID_ARG) return 12;
    {   /* injected allocation failure: create returns before touching a device */
        rtv_cache* c = NULL;
        setenv("RTV_INJECT_ALLOC_FAILURE", "1", 1);
        if (rtv_cache_create(&good[0], NULL, 0, &c) != RTV_ERR_OOM || c) return 13;
        unsetenv("RTV_INJECT_ALLOC_FAILURE");
        if (rtv_cache_create(&good[0], (void*)16, 8, &c) != RTV_ERR_INVALID_ARG) return 14;   /* too small */
        if (rtv_cache_create(NULL, NULL, 0, &c) != RTV_ERR_INVALID_ARG) return 15;
    }
    /* NULL handles everywhere */
    if (rtv_cache_destroy(NULL) != RTV_ERR_INVALID_ARG) return 16;
    if (rtv_cache_advance(NULL) != RTV_ERR_INVALID_ARG) return 17;
    if (rtv_attend(NULL, 0, NULL, 0, NULL) != RTV_ERR_INVALID_ARG) return 18;
    if (rtv_attend_static_scratch(NULL, 0, NULL, 0, NULL) != RTV_ERR_INVALID_ARG) return 19;
    if (rtv_cache_append(NULL, 0, NULL, NULL, NULL, 1, NULL) != RTV_ERR_INVALID_ARG) return 20;
    if (rtv_poll_error(NULL) != RTV_ERR_INVALID_ARG) return 21;
    if (rtv_cache_get_state(NULL, NULL) != RTV_ERR_INVALID_ARG) return 22;
    if (rtv_cache_export(NULL, 0, 0, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != RTV_ERR_INVALID_ARG) return 23;
    if (rtv_step_graph_launch(NULL, NULL) != RTV_ERR_INVALID_ARG) return 24;
    if (rtv_step_graph_destroy(NULL) != RTV_ERR_INVALID_ARG) return 25;
    if (rtv_step_graph_create(NULL, 1, NULL, NULL, NULL, NULL, 0, NULL, NULL) != RTV_ERR_INVALID_ARG) return 26;
    printf("host driver ok\n");
    return 0;
}
