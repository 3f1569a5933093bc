"""The boundary is a C ABI: a plain C99 program must compile against
include/fp4q.h (with warnings as errors), link libfp4q.so and get the
documented status codes from argument checks, which run before any CUDA call,
so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fp4q.h"

static int fails = 0;
#define EXPECT(call, want) do { fp4q_status s_ = (call); \
    if (s_ != (want)) { printf("FAIL %s -> %d, want %d\n", #call, (int)s_, (int)(want)); ++fails; } } while (0)

int main(void)
{
    static unsigned char buf[4096] __attribute__((aligned(16)));
    void* p = buf;
    float* f = (float*)buf;
    uint8_t* u8 = buf;
    int32_t* st = (int32_t*)buf;
    if (fp4q_version() < 10000) { printf("FAIL version\n"); ++fails; }
    if (strcmp(fp4q_status_string(FP4Q_OK), "ok") != 0) { printf("FAIL status string\n"); ++fails; }
    EXPECT(fp4q_global_absmax(p, FP4Q_BF16, -1, f, NULL, NULL), FP4Q_ERR_SHAPE);
    EXPECT(fp4q_global_absmax(p, FP4Q_BF16, 8, f, (int32_t*)(buf + 2), NULL), FP4Q_ERR_ALIGN);
    EXPECT(fp4q_nvfp4_sweepmse(p, (fp4q_dtype)7, 1, 16, f, u8, u8, f, NULL, NULL, st, NULL), FP4Q_ERR_DTYPE);
    EXPECT(fp4q_nvfp4_sweepmse(p, FP4Q_BF16, 1, 24, f, u8, u8, f, NULL, NULL, st, NULL), FP4Q_ERR_SHAPE);
    EXPECT(fp4q_nvfp4_sweepwmse(p, FP4Q_BF16, 1, 16, f, NULL, u8, u8, f, NULL, NULL, st, NULL), FP4Q_ERR_NULL);
    EXPECT(fp4q_mxfp4_quant(buf + 2, FP4Q_BF16, 1, 32, u8, u8, NULL, NULL, st, NULL), FP4Q_ERR_ALIGN);
    EXPECT(fp4q_mxfp4_quant_hadamard(p, FP4Q_F32, 1, 32, NULL, u8, u8, NULL, NULL, st, NULL), FP4Q_ERR_NULL);
    EXPECT(fp4q_nvfp4_sweep_dynamic(p, FP4Q_BF16, 1, 16, NULL, f, u8, u8, f, NULL, NULL, p,
                                    fp4q_dynamic_workspace_bytes() - 1, st, NULL), FP4Q_ERR_ARG);
    EXPECT(fp4q_focus_quant(FP4Q_NVFP4, p, FP4Q_BF16, 1, 16, u8, f, p, 12, u8, NULL, NULL, st, NULL), FP4Q_ERR_ARG);
    EXPECT(fp4q_nvfp4_gptq(f, 1, 16, f, f, u8, u8, f, NULL, p, 0, st, NULL), FP4Q_ERR_ARG);
    EXPECT(fp4q_scales_to_mma_layout(u8, -1, 4, u8, NULL), FP4Q_ERR_SHAPE);
    EXPECT(fp4q_dequant((fp4q_format)5, u8, u8, f, 1, 16, p, FP4Q_BF16, NULL), FP4Q_ERR_DTYPE);
    EXPECT(fp4q_mxfp4_unrotate(p, FP4Q_BF16, 1, 48, (const uint32_t*)buf, p, NULL), FP4Q_ERR_SHAPE);
    EXPECT(fp4q_probe_copy(p, buf + 1024, 24, NULL), FP4Q_ERR_SHAPE);
    EXPECT(fp4q_probe_copy(buf + 8, buf + 1024, 32, NULL), FP4Q_ERR_ALIGN);
    {
        fp4q_batch_tensor t;
        memset(&t, 0, sizeof(t));
        t.w = p; t.rows = 1; t.cols = 40;
        EXPECT(fp4q_mxfp4_quant_group(&t, 1, FP4Q_BF16, st, NULL), FP4Q_ERR_SHAPE);
        t.cols = 32;
        EXPECT(fp4q_nvfp4_sweep_group(&t, 1, FP4Q_BF16, st, NULL), FP4Q_ERR_NULL);
        EXPECT(fp4q_nvfp4_sweep_group(&t, -1, FP4Q_BF16, st, NULL), FP4Q_ERR_SHAPE);
        EXPECT(fp4q_mxfp4_quant_group(&t, 0, FP4Q_BF16, NULL, NULL), FP4Q_OK);
        if (FP4Q_GROUP_MAX < 8) { printf("FAIL group max\n"); ++fails; }
    }
    if (fp4q_mma_scale_bytes(130, 6) != 2 * 2 * 512) { printf("FAIL mma bytes\n"); ++fails; }
    if (fp4q_gptq_workspace_bytes(5) != 2 * 8 * 128 * 4) { printf("FAIL gptq workspace\n"); ++fails; }
    printf(fails ? "failed\n" : "ok\n");
    return fails != 0;
}
"""


@pytest.fixture(scope="module")
def lib():
    from fp4_post_weight_grid_b200 import build
    return build.build()


def test_c99_program_against_the_header(lib, tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           "-L", libdir, "-lfp4q", "-Wl,-rpath," + libdir, "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip().endswith("ok"), run.stdout + run.stderr
