"""The bounds-checked build on a cross-section of the GPU parity cases.

``libfp4moe_checked.so`` is the library compiled with -DMOE_DEBUG_CHECKS:
every index a kernel reads from device data (routing target, location-table
entry, padded row's token or pair) is checked before use, and a bad one is
recorded in the layer's error word instead of faulting.  A child process that
loads it (FP4MOE_CHECKED=1) runs parity cases that reach every kernel --
MXFP4 tensor-core tiles of both sizes, the NVFP4 register and tensor-core
paths, INT4 / FP8 experts, A4, both shared-expert kernels, router variants,
staged waves and the residency policies -- and each of them must match the
oracle with no check firing (every run asserts a zero error word).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = ("small_layers_full_parity or olmoe_decode_full_parity or qwen3_30b_like_paged "
         "or format_parity or format_paged or nvfp4_prefill_tensor_core_parity "
         "or a4_small_layers or a4_paged or variant_paged or router_variant_parity or policy "
         "or bounded_waits")

FILES = ["tests/test_gpu_parity.py", "tests/test_gpu_formats.py", "tests/test_gpu_nv_tc.py",
         "tests/test_gpu_a4.py", "tests/test_gpu_variants.py", "tests/test_gpu_policy.py"]

PROBE = r"""
import synth, fp4_expert_layer_b200 as F
from fp4_expert_layer_b200 import _lib
from tests import _gpu as G
wl = synth.workload("tiny")
layer = G.make_layer(synth.make_layer(wl), max_tokens=4)
G.run(layer, synth.make_tokens(wl, 4))
layer.close()
maps = open("/proc/self/maps").read()
assert _lib.SO.endswith("libfp4moe_checked.so"), _lib.SO
assert "libfp4moe_checked.so" in maps and "libfp4moe.so" not in maps
print("checked library loaded")
"""


@pytest.mark.gpu
def test_checked_build_passes_a_parity_cross_section():
    from fp4_expert_layer_b200 import build
    build.build(checked=True)
    env = dict(os.environ, FP4MOE_CHECKED="1")
    r = subprocess.run([sys.executable, "-c", PROBE], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "checked library loaded" in r.stdout, r.stdout[-2000:] + r.stderr[-3000:]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", *FILES, "-k", CASES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = r.stdout[-4000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail
