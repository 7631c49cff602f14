"""Writes tmem_io.cuh: the tcgen05.ld / tcgen05.st wrappers (32x32b shape) the
kernels use to move accumulator columns between TMEM and registers.

Each wrapper is one inline-asm block whose operand lists are long and regular
(one "=r"/"r" per 32-bit column), so they are generated rather than typed:

    python rank_biased_window_b200/csrc/gen_tmem_io.py          # rewrite the header
    python rank_biased_window_b200/csrc/gen_tmem_io.py --check  # exit 1 if it differs

A .x32 instruction moves 32 columns; wider transfers issue several of them and
wait once.  tests/test_abi.py checks that the committed header is this
script's output.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
OUT = os.path.join(HERE, "tmem_io.cuh")


def _regs(first, n):
    return ", ".join(f"%{first + i}" for i in range(n))


def _outs(n):
    return ", ".join(f'"=r"(r[{i}])' for i in range(n))


def _ins(n):
    return ", ".join(f'"r"(r[{i}])' for i in range(n))


def ld(ncols):
    """tmem_ld<ncols>: ncols consecutive columns, then one wait."""
    if ncols == 16:
        body = [f'"tcgen05.ld.sync.aligned.32x32b.x16.b32 {{{_regs(0, 16)}}}, [%16];\\n"']
        addrs = ['"r"(taddr + 0u)']
        how = "1 x .x16"
    else:
        n32 = ncols // 32
        body = [f'"tcgen05.ld.sync.aligned.32x32b.x32.b32 {{{_regs(32 * j, 32)}}}, [%{ncols + j}];\\n"'
                for j in range(n32)]
        addrs = [f'"r"(taddr + {32 * j}u)' for j in range(n32)]
        how = f"{n32} x .x32"
    lines = [
        f"// Loads {ncols} consecutive 32-bit TMEM columns of this thread's lane",
        f"// (32x32b shape, {how}) and waits for them.",
        f"__device__ __forceinline__ void tmem_ld{ncols}(uint32_t taddr, uint32_t (&r)[{ncols}]) {{",
        "  asm volatile(",
    ]
    lines += [f"      {b}" for b in body]
    lines += [
        '      "tcgen05.wait::ld.sync.aligned;\\n"',
        f"      : {_outs(ncols)}",
        f"      : {', '.join(addrs)}",
        '      : "memory");',
        "}",
        "",
    ]
    return lines


def st(ncols):
    """tmem_st<ncols>: ncols consecutive columns, then one wait."""
    if ncols <= 32:
        body = [f'"tcgen05.st.sync.aligned.32x32b.x{ncols}.b32 [%0], {{{_regs(1, ncols)}}};\\n"']
        addrs = ['"r"(taddr + 0u)']
    else:
        n32 = ncols // 32
        body = [f'"tcgen05.st.sync.aligned.32x32b.x32.b32 [%{j}], {{{_regs(n32 + 32 * j, 32)}}};\\n"'
                for j in range(n32)]
        addrs = [f'"r"(taddr + {32 * j}u)' for j in range(n32)]
    lines = [
        f"// Stores {ncols} consecutive 32-bit TMEM columns of this thread's lane",
        "// (32x32b shape) and waits until the stores have completed.",
        f"__device__ __forceinline__ void tmem_st{ncols}(uint32_t taddr, const uint32_t (&r)[{ncols}]) {{",
        "  asm volatile(",
    ]
    lines += [f"      {b}" for b in body]
    lines += [
        '      "tcgen05.wait::st.sync.aligned;\\n"',
        "      :",
        f"      : {', '.join(addrs)}, {_ins(ncols)}",
        '      : "memory");',
        "}",
        "",
    ]
    return lines


def ld_multi(names, comment, sig):
    """32 columns from each of len(names) addresses, one wait."""
    n = len(names)
    lines = comment + [sig, "  asm volatile("]
    lines += [f'      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {{{_regs(32 * j, 32)}}}, [%{32 * n + j}];\\n"'
              for j in range(n)]
    lines += [
        '      "tcgen05.wait::ld.sync.aligned;\\n"',
        f"      : {_outs(32 * n)}",
        f"      : {', '.join(f'\"r\"({a})' for a in names)}",
        '      : "memory");',
        "}",
        "",
    ]
    return lines


def header():
    out = [
        "// tcgen05.ld / tcgen05.st wrappers, 32x32b shape: thread t of warp w owns",
        "// TMEM lane 32*(w%4)+t; register i holds column (taddr.col + i).",
        "// Written by gen_tmem_io.py in this directory: change the generator, then",
        "// rerun it, rather than editing this file.",
        "#pragma once",
        "#include <cstdint>",
        "",
        "namespace rfb {",
        "",
    ]
    for n in (16, 32, 64, 128):
        out += ld(n)
    for n in (16, 32, 64):
        out += st(n)
    out += ld_multi(
        ["taddr_a", "taddr_b"],
        ["// Loads 32 columns at taddr_a into r[0..31] and 32 columns at taddr_b into",
         "// r[32..63] (32x32b shape), then waits once for both."],
        "__device__ __forceinline__ void tmem_ld32x2(uint32_t taddr_a, uint32_t taddr_b, "
        "uint32_t (&r)[64]) {")
    out += [
        "// tcgen05.st of 16 columns without waiting; pair with tmem_st_wait().",
        "__device__ __forceinline__ void tmem_st16_nowait(uint32_t taddr, const uint32_t (&r)[16]) {",
        "  asm volatile(",
        f'      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {{{_regs(1, 16)}}};\\n"',
        "      :",
        f'      : "r"(taddr), {_ins(16)}',
        '      : "memory");',
        "}",
        "// Waits until all prior tcgen05.st of this thread have completed.",
        "__device__ __forceinline__ void tmem_st_wait() {",
        '  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");',
        "}",
        "",
    ]
    out += ld_multi(
        ["ta", "tb", "tc", "td"],
        ["// Loads 32 columns at each of four addresses into r[0..31], r[32..63],",
         "// r[64..95], r[96..127] (32x32b shape), then waits once."],
        "__device__ __forceinline__ void tmem_ld32x4(uint32_t ta, uint32_t tb, uint32_t tc, "
        "uint32_t td,\n                                            uint32_t (&r)[128]) {")
    out += ["}  // namespace rfb", ""]
    return "\n".join(out)


if __name__ == "__main__":
    text = header()
    if "--check" in sys.argv:
        with open(OUT) as f:
            sys.exit(0 if f.read() == text else 1)
    with open(OUT, "w") as f:
        f.write(text)
    print(OUT)
