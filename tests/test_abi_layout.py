"""The binding's ctypes argument structs have the layout of include/msc.h:
a small C program built with the host compiler prints sizeof and offsetof of
every field the binding names, and they must agree (a field the header lacks
fails the build).  CPU only."""
import ctypes
import os
import subprocess

import pytest

from selective_state_space_14_b200 import msc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PAIRS = [("msc_ss_fwd_args", msc.SsFwdArgs), ("msc_ss_conv_args", msc.SsConvArgs),
         ("msc_ss_bwd_args", msc.SsBwdArgs), ("msc_su_args", msc.SuArgs),
         ("msc_m3_fwd_args", msc.M3FwdArgs), ("msc_m3_bwd_args", msc.M3BwdArgs),
         ("msc_m3_su_args", msc.M3SuArgs), ("msc_m3_disc_step_args", msc.M3DiscStepArgs),
         ("msc_m3_disc_args", msc.M3DiscArgs), ("msc_m3_disc_bwd_args", msc.M3DiscBwdArgs),
         ("msc_conv_fwd_args", msc.ConvFwdArgs), ("msc_conv_bwd_args", msc.ConvBwdArgs),
         ("msc_m3_raw_args", msc.M3RawArgs), ("msc_m3_raw_grads", msc.M3RawGrads)]


def test_every_header_struct_is_bound():
    import re
    text = open(os.path.join(ROOT, "include", "msc.h")).read()
    assert sorted(re.findall(r"^\} (msc_\w+_(?:args|grads));", text, flags=re.M)) == \
        sorted(c for c, _ in PAIRS)


def test_struct_layouts_match_the_header(tmp_path):
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "msc.h"', 'int main(void) {']
    for cname, cls in PAIRS:
        lines.append(f'  printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    try:
        subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                        str(exe)], check=True, capture_output=True, text=True)
    except FileNotFoundError:
        pytest.skip("no host C compiler")
    except subprocess.CalledProcessError as e:
        raise AssertionError(e.stderr)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True,
                               text=True).stdout.splitlines():
        cname, field, val = line.split()
        got[(cname, field)] = int(val)
    for cname, cls in PAIRS:
        assert got[(cname, "sizeof")] == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert got[(cname, fname)] == getattr(cls, fname).offset, (cname, fname)
