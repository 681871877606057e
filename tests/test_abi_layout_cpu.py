"""The Python binding's descriptor must have the C struct's layout: every
field of kvq_cache_desc at the same offset and the same total size, read from
include/kvq.h by the host C compiler (no GPU)."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import kv_cache_mixed_kvq_b200 as kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FIELDS = [name for name, _ in kvq.KvqCacheDesc._fields_]


def _c_layout():
    src = ['#include <stddef.h>', '#include <stdio.h>', '#include "kvq.h"', 'int main(void) {',
           '  printf("size %zu\\n", sizeof(kvq_cache_desc));']
    for f in FIELDS:
        src.append(f'  printf("{f} %zu\\n", offsetof(kvq_cache_desc, {f}));')
    src += ['  return 0;', '}']
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        with open(c, "w") as fh:
            fh.write("\n".join(src) + "\n")
        subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        out = subprocess.check_output([exe], text=True)
    return dict((k, int(v)) for k, v in (line.split() for line in out.splitlines()))


def test_descriptor_layout_matches_the_header():
    try:
        layout = _c_layout()
    except (OSError, subprocess.CalledProcessError) as e:  # no host compiler
        pytest.skip(f"gcc unavailable: {e}")
    assert layout.pop("size") == ctypes.sizeof(kvq.KvqCacheDesc)
    for name in FIELDS:
        assert layout[name] == getattr(kvq.KvqCacheDesc, name).offset, name
