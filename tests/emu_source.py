"""Maps the CUDA source of the library's kernels to source the CPU block emulator
(tests/emu/enc/block_emu.h) compiles: inline PTX becomes host atomics and copies,
and `__shared__` variables become per-block storage."""

import re


def host_source(text: str) -> str:
    """The device source with its inline PTX and shared-memory declarations mapped to
    the emulator's calls."""
    reps = [
        (r'asm volatile\("cp\.async\.cg\.shared\.global \[%0\], \[%1\], 16;\\n" ::"r"\((\w+)\), "l"\((\w+)\)\s*:\s*"memory"\);',
         r"emu_cp16(\1, \2);"),
        (r'asm volatile\("cp\.async\.cg\.shared\.global \[%0\], \[%1\], 16, %2;\\n" ::"r"\((\w+)\), "l"\((\w+)\), '
         r'"r"\((\w+)\)\s*:\s*"memory"\);', r"emu_cp16z(\1, \2, \3);"),
        (r'asm volatile\("cp\.async\.ca\.shared\.global \[%0\], \[%1\], 4;\\n" ::"r"\((\w+)\), "l"\((\w+)\)\s*:\s*"memory"\);',
         r"emu_cp4(\1, \2);"),
        (r'asm volatile\("cp\.async\.commit_group;\\n" ::: "memory"\);', ";"),
        (r'asm volatile\("cp\.async\.wait_all;\\n" ::: "memory"\);', ";"),
        (r'asm volatile\("st\.release\.gpu\.global\.u64 \[%0\], %1;" ::"l"\(p\), "l"\(v\) : "memory"\);',
         "__atomic_store_n(p, v, __ATOMIC_RELEASE);"),
        (r'asm volatile\("ld\.acquire\.gpu\.global\.u64 %0, \[%1\];" : "=l"\(v\) : "l"\(p\) : "memory"\);',
         "v = __atomic_load_n(p, __ATOMIC_ACQUIRE);"),
        (r'asm volatile\("ld\.relaxed\.gpu\.global\.u64 %0, \[%1\];" : "=l"\(v\) : "l"\(p\) : "memory"\);',
         "v = __atomic_load_n(p, __ATOMIC_RELAXED);"),
        (r'asm volatile\("ld\.acquire\.gpu\.global\.u32 %0, \[%1\];" : "=r"\(v\) : "l"\(p\) : "memory"\);',
         "v = __atomic_load_n(p, __ATOMIC_ACQUIRE);"),
        (r'asm volatile\("prefetch\.global\.L2 \[%0\];" ::"l"\([^;]*\);', ";"),
        (r"extern __shared__ __align__\(16\) uint32_t smem\[\];",
         "uint32_t* smem = reinterpret_cast<uint32_t*>(emu_smem());"),
        (r"__shared__ __align__\(16\) ", "__shared__ "),
        (r"__shared__\s+([\w:<> ]+?)\s+(\w+)\s*(\[[^\]]*\])?\s*;", r"auto& \2 = emu_shared<\1\3>(__LINE__);"),
    ]
    for pat, rep in reps:
        text = re.sub(pat, rep, text)
    assert "asm" not in text and "__shared__" not in text
    return text
