"""Host builds of libpivot's CUDA sources for the CPU tests (test
infrastructure).  The CUDA features the kernels use are emulated by
tests/emu (one host thread per CUDA thread, block barriers, warp
collectives, dynamic shared memory filled with junk); the kernel sources are
used as they are, with only their launch syntax and shared-memory
declarations rewritten, and the few helpers they take from common.cuh are
copied from there verbatim."""
import re
import shutil
import subprocess
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]
CSRC = ROOT / "top_token_selection_b200" / "csrc"
EMU = ROOT / "tests" / "emu"

# Device helpers the proxy / CUDA-core sources use beyond emu.h: IEEE single
# operations with round to nearest (the host's default), bf16 widening; the
# bf16 and e4m3 narrowing conversions are not emulated and abort if reached.
EXTRA = r"""
struct alignas(16) uint4 { uint32_t x, y, z, w; };
inline uint4 make_uint4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) { return {a, b, c, d}; }
inline float __fadd_rn(float a, float b) { return a + b; }
inline float __fmul_rn(float a, float b) { return a * b; }
inline float __fdiv_rn(float a, float b) { return a / b; }
inline float fmaf(float a, float b, float c) { return std::fma(a, b, c); }
struct __nv_bfloat16 { uint16_t x; };
inline __nv_bfloat16 __float2bfloat16_rn(float) { EMU_FAIL("bf16 store not emulated"); }
inline uint16_t __bfloat16_as_ushort(__nv_bfloat16 v) { return v.x; }
inline float e4m3_to_f32(uint8_t) { EMU_FAIL("e4m3 not emulated"); }
inline uint8_t f32_to_e4m3_satfinite(float) { EMU_FAIL("e4m3 not emulated"); }
inline float bf16_to_f32(uint16_t c) { return __uint_as_float((uint32_t)c << 16); }
"""


def rewrite(src, pairs):
    """Exact one-time replacements (fails loudly when the source changed shape)."""
    for old, new in pairs:
        assert src.count(old) == 1, f"kernel source changed shape: {old!r}"
        src = src.replace(old, new)
    return src


def rewrite_launches(src):
    """kernel<<<grid, block, smem, stream>>>(args); -> emu_launch(grid, block, smem, [&] {...});"""
    pat = re.compile(r"([A-Za-z_][\w]*(?:<[^<>;]*>)?)<<<(.*?),(.*?),(.*?),\s*stream>>>\((.*?)\);",
                     re.S)
    out, n = pat.subn(lambda m: f"emu_launch({m.group(2)}, {m.group(3)}, {m.group(4)}, "
                                f"[&] {{ {m.group(1)}({m.group(5)}); }});", src)
    assert n == src.count("<<<"), "a launch was not rewritten"
    return out


def prepare(d: Path, extra=False):
    """Write the emulation headers into d: common.cuh (the error bits and key
    helpers copied from the real one), kernels.h and segments.h."""
    common = (CSRC / "common.cuh").read_text()
    errbits = re.search(r"enum : uint32_t \{.*?\};", common, re.S).group(0)
    # the debug-build checks (used as they are; on when compiled with PIVOT_DEBUG)
    checks = re.search(r"#ifdef PIVOT_DEBUG\n.*?#endif\n", common, re.S).group(0)
    helpers = re.search(r"// Order-preserving unsigned key.*?int ceil_div\(int a, int b\) \{[^}]*\}",
                        common, re.S).group(0)
    (d / "common.cuh").write_text(
        "#pragma once\n#include <cmath>\n#include \"emu.h\"\n#include \"pivot.h\"\n"
        "namespace pivot {\n" + errbits + "\nextern uint32_t g_error_word;\n"
        "inline void raise_error(uint32_t bit) { __atomic_fetch_or(&g_error_word, bit, "
        "__ATOMIC_SEQ_CST); }\n" + checks + helpers + (EXTRA if extra else "") +
        "\n}  // namespace pivot\n")
    kernels = rewrite((CSRC / "kernels.h").read_text(),
                      [("#include <cuda.h>", "#include \"emu.h\""), ("#include <cuda_runtime.h>\n", "")])
    (d / "kernels.h").write_text(kernels)
    shutil.copy(CSRC / "segments.h", d / "segments.h")


def compile_(d: Path, sources, out: Path, shared=False, sanitize=False, defines=()):
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-pthread", "-ffp-contract=off",
           "-I", str(d), "-I", str(EMU), "-I", str(ROOT / "include")]
    cmd += [f"-D{x}" for x in defines]
    if shared:
        cmd += ["-fPIC", "-shared"]
    if sanitize:
        cmd += ["-fsanitize=address,undefined", "-fno-sanitize-recover=all"]
    res = subprocess.run(cmd + [str(EMU / "emu.cpp"), *map(str, sources), "-o", str(out)],
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-4000:]
    return out
