"""The boundary from plain C: a C11 program includes include/nomas.h, links
libnomas.so and drives the calls that need no GPU (descriptor reset and state
checks, the evicted-frame range, host-side argument errors, status strings).
Nothing here goes through Python or PyTorch; device pointers are fake
addresses that the host-side checks never dereference."""

import os
import subprocess

import pytest

import segment_causal_kv_b200 as nm
from segment_causal_kv_b200 import build as nm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#include "nomas.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAIL line %d: %s\n", __LINE__, #cond); return 1; } } while (0)

int main(void) {
    nomas_cache c;
    memset(&c, 0, sizeof c);
    c.mode = NOMAS_CACHE_INT8;
    c.heads = 16;
    c.head_dim = NOMAS_HEAD_DIM;
    c.grid_h = 22;
    c.grid_w = 40;
    c.window_frames = 18;
    c.capacity_frames = 18;
    c.rope_theta = 256.0f;
    c.k = (void *)(uintptr_t)0x7F0000000000ull;
    c.v = (void *)(uintptr_t)0x7F0040000000ull;
    c.k_scale = (float *)(uintptr_t)0x7F0080000000ull;
    c.v_scale = (float *)(uintptr_t)0x7F00C0000000ull;

    /* a descriptor that was never reset is refused */
    int32_t count = -1;
    int64_t first = -1;
    CHECK(nomas_kv_evicted_frames(&c, 3, &count, &first) == NOMAS_ERR_STATE);
    CHECK(nomas_cache_reset(&c) == NOMAS_OK);
    CHECK(c.frames_committed == 0 && c.valid_frames == 0 && c.head_slot == 0 && c.check != 0);

    /* an empty window drops nothing; a full one drops its oldest frames */
    CHECK(nomas_kv_evicted_frames(&c, 3, &count, &first) == NOMAS_OK && count == 0);
    c.frames_committed = 24; c.valid_frames = 18; c.head_slot = 6;  /* frames 6..23 held */
    CHECK(nomas_kv_evicted_frames(&c, 3, &count, &first) == NOMAS_OK && count == 3 && first == 6);
    CHECK(nomas_kv_evicted_frames(&c, 40, &count, &first) == NOMAS_OK && count == 18 && first == 6);

    /* host-side argument checks, before any device work */
    CHECK(nomas_kv_commit(&c, c.k, c.v, 16 * 128, -1, NULL) == NOMAS_ERR_ARG);
    CHECK(nomas_kv_commit(&c, c.k, c.v, 16 * 128 - 8, 3, NULL) == NOMAS_ERR_ARG);
    CHECK(nomas_kv_commit(&c, c.k, c.v, 16 * 128, 0, NULL) == NOMAS_OK);
    CHECK(nomas_camera_attn(c.k, 16 * 128, 3, 880, 16, c.k, c.v, 0, 1, c.v, 16 * 128, NULL) == NOMAS_ERR_ARG);
    CHECK(nomas_camera_attn(c.k, 16 * 128, 0, 880, 16, c.k, c.v, 1, 1, c.v, 16 * 128, NULL) == NOMAS_OK);
    CHECK(nomas_seg_attn_workspace_bytes(&c, 3, 256) >= nomas_seg_attn_workspace_min_bytes(&c, 3, 256));
    CHECK(nomas_seg_attn_workspace_min_bytes(&c, 3, 256) > 0);

    /* a configuration changed after the reset is caught */
    c.grid_w = 41;
    CHECK(nomas_kv_evicted_frames(&c, 3, &count, &first) == NOMAS_ERR_STATE);
    CHECK(nomas_seg_attn_workspace_bytes(&c, 3, 256) == 0);

    CHECK(strcmp(nomas_status_string(NOMAS_OK), "NOMAS_OK") == 0);
    CHECK(strncmp(nomas_status_string(NOMAS_ERR_CAPACITY), "NOMAS_ERR_CAPACITY", 18) == 0);
    printf("ok\n");
    return 0;
}
"""


def test_plain_c_client_links_and_drives_the_host_side(tmp_path):
    nm_build.build()
    src = tmp_path / "client.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "client"
    libdir = os.path.dirname(nm.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-L", libdir, "-l:libnomas.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
