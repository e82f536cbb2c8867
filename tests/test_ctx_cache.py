"""Host test of the context-keyed caches in csrc/ctx_cache.h (no GPU).

The library caches, per device, the device address of its fault word, the address of the
no-alloc GEMM's fixed scratch buffer and each kernel's shared-memory opt-in.  All three
belong to the CUDA context the module was loaded in, so after a device reset they must be
looked up again.  The cache is keyed on the context id; this test compiles the header with
the host C++ compiler and drives it with fake ids and a fake lookup.
"""
import os
import shutil
import subprocess
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_gemv_rabit_b200", "csrc")

PROGRAM = textwrap.dedent(r"""
    #include <cstdio>
    #include "ctx_cache.h"

    static int lookups = 0;
    static int next_address = 1000;
    // fake symbol lookup: a new address each time, as after a module reload
    static int lookup(long *out) { ++lookups; *out = next_address++; return 0; }
    static int failing(long *out) { (void)out; ++lookups; return 7; }

    int main() {
        rabit::ContextCache<long> cache;
        long v = 0;
        int bad = 0;
        // first use in context 11 on device 0: one lookup
        bad |= cache.get(0, 11, lookup, &v) != 0 || v != 1000 || lookups != 1;
        // same context: served from the cache
        bad |= cache.get(0, 11, lookup, &v) != 0 || v != 1000 || lookups != 1;
        // another device keeps its own entry
        bad |= cache.get(1, 11, lookup, &v) != 0 || v != 1001 || lookups != 2;
        // the context of device 0 was reset: id 12 refills with the new address
        bad |= cache.get(0, 12, lookup, &v) != 0 || v != 1002 || lookups != 3;
        bad |= cache.get(0, 12, lookup, &v) != 0 || v != 1002 || lookups != 3;
        // id 0 (no context could be read) always looks up again
        bad |= cache.get(0, 0, lookup, &v) != 0 || v != 1003 || lookups != 4;
        bad |= cache.get(0, 0, lookup, &v) != 0 || v != 1004 || lookups != 5;
        // a failed lookup reports its status and leaves the entry empty
        bad |= cache.get(2, 13, failing, &v) != 7 || lookups != 6;
        bad |= cache.get(2, 13, lookup, &v) != 0 || v != 1005 || lookups != 7;
        // devices past the table are never cached
        bad |= cache.get(64, 13, lookup, &v) != 0 || v != 1006 || lookups != 8;
        bad |= cache.get(64, 13, lookup, &v) != 0 || v != 1007 || lookups != 9;

        rabit::ContextFlags flags;
        bad |= flags.done(0, 11);
        flags.mark(0, 11);
        bad |= !flags.done(0, 11);
        bad |= flags.done(0, 12);      // new context: the setting must be made again
        bad |= flags.done(1, 11);      // other device
        bad |= flags.done(0, 0);       // unknown context never counts as done
        flags.mark(0, 12);
        bad |= !flags.done(0, 12) || flags.done(0, 11);
        std::printf("%s %d\n", bad ? "FAIL" : "OK", lookups);
        return bad;
    }
""")


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_context_keyed_cache_refills_after_context_change(tmp_path):
    src = tmp_path / "ctx_cache_test.cpp"
    exe = tmp_path / "ctx_cache_test"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe), "-pthread"],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.startswith("OK"), out.stdout + out.stderr
