"""The Python binding's ctypes structures and constants match the C header: a probe built
from include/tre.h with the host compiler prints every field's offset and size and every
constant, and each must equal what the binding declares.  CPU only."""
import ctypes
import os
import shutil
import subprocess

import pytest

from persistent_tile_pipelined_b200 import tre

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BUILD = os.path.join(ROOT, "tests", "_build")

CONSTANTS = ["TRE_OK", "TRE_ERR_INVALID_ARG", "TRE_ERR_CUDA", "TRE_ERR_OCCUPANCY",
             "TRE_ERR_DEP_TIMEOUT", "TRE_ERR_POS_RANGE", "TRE_ERR_UNSUPPORTED", "TRE_ERR_BOUNDS",
             "TRE_ERR_STATE", "TRE_LAYER_GQA", "TRE_LAYER_MLA", "TRE_LAYER_MOE",
             "TRE_DEBUG_HIDDEN", "TRE_DEBUG_TRACE", "TRE_DEBUG_FAULT_INJECT",
             "TRE_DEBUG_NO_OVERLAP", "TRE_W_SLOTS", "TRE_LAUNCH_PERSISTENT", "TRE_LAUNCH_PER_OP",
             "TRE_WEIGHTS_BF16", "TRE_WEIGHTS_FP8_BLOCK128", "TRE_WEIGHTS_FP4_EXPERTS"]


def probe_source():
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "tre.h"', 'int main(void) {']
    for st in (tre.tre_config, tre.tre_weights, tre.tre_plan_info):
        name = st.__name__
        lines.append(f'  printf("{name}:size %zu\\n", sizeof({name}));')
        for field, _ in st._fields_:
            lines.append(f'  printf("{name}.{field} %zu %zu\\n", offsetof({name}, {field}), '
                         f'sizeof((({name}*)0)->{field}));')
    for c in CONSTANTS:
        lines.append(f'  printf("{c} %d\\n", (int)({c}));')
    lines += ['  return 0;', '}']
    return "\n".join(lines) + "\n"


@pytest.fixture(scope="module")
def probe():
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    os.makedirs(BUILD, exist_ok=True)
    src, exe = os.path.join(BUILD, "abi_probe.c"), os.path.join(BUILD, "abi_probe")
    with open(src, "w") as f:
        f.write(probe_source())
    subprocess.check_call([cc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           src, "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    vals = {}
    for line in out.splitlines():
        key, *nums = line.split()
        vals[key] = tuple(int(x) for x in nums)
    return vals


@pytest.mark.parametrize("st", [tre.tre_config, tre.tre_weights, tre.tre_plan_info],
                         ids=lambda s: s.__name__)
def test_struct_layout_matches_the_header(probe, st):
    name = st.__name__
    assert probe[f"{name}:size"] == (ctypes.sizeof(st),)
    for field, ctype in st._fields_:
        desc = getattr(st, field)
        assert probe[f"{name}.{field}"] == (desc.offset, ctypes.sizeof(ctype)), field


def test_constants_match_the_header(probe):
    for c in CONSTANTS:
        assert probe[c] == (getattr(tre, c),), c
