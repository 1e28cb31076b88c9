"""The ctypes mirror of the C ABI matches the header as a C compiler lays it
out: every field offset and the size of ta_params and ta_plan_views, and the
values of the status, format, tier and debug constants.  A drift between the
two would hand the library shifted fields without any error, so the header is
compiled here with the host C compiler and its layout compared with the
binding's."""

import ctypes
import os
import shutil
import subprocess

import pytest

from precision_attention_video_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CONSTANTS = ["TA_OK", "TA_ERR_INVALID_ARG", "TA_ERR_UNSUPPORTED", "TA_ERR_WORKSPACE",
             "TA_ERR_CUDA", "TA_ERR_TIMEOUT", "TA_LOW_NONE", "TA_LOW_FP8_E4M3", "TA_LOW_NVFP4",
             "TA_LOW_NVFP4_RES", "TA_TIER_SKIP", "TA_TIER_LOW", "TA_TIER_RES", "TA_TIER_FULL",
             "TA_DEBUG_DROP_FIRST_K"]


def _c_layout(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "tiered_attn.h"',
             'int main(void) {']
    for struct, cls in (("ta_params", B.ta_params), ("ta_plan_views", B.ta_plan_views)):
        lines.append(f'  printf("sizeof {struct} %zu\\n", sizeof({struct}));')
        for name, _ in cls._fields_:
            lines.append(f'  printf("offset {struct}.{name} %zu\\n", offsetof({struct}, {name}));')
    for c in CONSTANTS:
        lines.append(f'  printf("const {c} %d\\n", (int)({c}));')
    lines.append('  return 0;\n}')
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = {}
    for line in out.splitlines():
        kind, key, val = line.split()
        got[(kind, key)] = int(val)
    return got


def test_struct_layout_and_constants_match_the_header(tmp_path):
    got = _c_layout(tmp_path)
    for struct, cls in (("ta_params", B.ta_params), ("ta_plan_views", B.ta_plan_views)):
        assert got[("sizeof", struct)] == ctypes.sizeof(cls), struct
        for name, _ in cls._fields_:
            assert got[("offset", f"{struct}.{name}")] == getattr(cls, name).offset, (struct, name)
    for c in CONSTANTS:
        assert got[("const", c)] == getattr(B, c), c


def test_header_compiles_as_c_and_as_cpp(tmp_path):
    # the header is the product's boundary: plain C99 and C++ callers both
    # include it without warnings
    for cc, std, ext in (("gcc", "-std=c99", "c"), ("g++", "-std=c++17", "cpp")):
        exe = shutil.which(cc)
        if exe is None:
            pytest.skip(f"no {cc}")
        src = tmp_path / f"inc.{ext}"
        src.write_text('#include "tiered_attn.h"\nint main(void) { ta_params p; (void)p; return 0; }\n')
        subprocess.run([exe, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                        os.path.join(ROOT, "include"), str(src), "-o", str(tmp_path / "inc")],
                       check=True, capture_output=True)


def test_default_tier_costs_agree_between_header_oracle_and_calibration(tmp_path):
    # the price router's default costs are stated twice, independently: in
    # the header (what the library uses when tier_cost is all zero) and in the
    # oracle; the stored price was calibrated with them
    import json

    from latent_gen import get_config
    from oracle import route as R
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    names = ["SKIP", "FP8", "NVFP4", "NVFP4_RES", "FULL"]
    src = tmp_path / "cost.c"
    src.write_text('#include <stdio.h>\n#include "tiered_attn.h"\nint main(void) {\n' +
                   "".join(f'  printf("%.17g\\n", (double)TA_TIER_COST_{n});\n' for n in names) +
                   "  return 0;\n}\n")
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(tmp_path / "cost")], check=True, capture_output=True)
    out = subprocess.run([str(tmp_path / "cost")], check=True, capture_output=True, text=True).stdout
    c = dict(zip(names, (float(x) for x in out.split())))
    for low, low_cost in ((B.TA_LOW_FP8_E4M3, c["FP8"]), (B.TA_LOW_NVFP4, c["NVFP4"]),
                          (B.TA_LOW_NVFP4_RES, c["NVFP4"])):
        assert R.default_tier_cost(low) == (c["SKIP"], low_cost, c["NVFP4_RES"], c["FULL"]), low
    with open(os.path.join(ROOT, "latent_gen", "price.json")) as f:
        stored = json.load(f)
    cfg = get_config("480p-price")
    assert tuple(stored["tier_cost"]) == R.default_tier_cost(cfg.low)
    assert stored["price"] == cfg.price and not any(cfg.tier_cost)
