"""Writes tmem_ldst.cuh: the long but regular operand lists of the TMEM load/store wrappers."""
import os

def ld(n):
    outs = ", ".join(f"%{i}" for i in range(n))
    cons = ", ".join(f'"=r"(r[{i}])' for i in range(n))
    return f'''// Loads {n} consecutive 32-bit TMEM columns of this warp's 32 lanes (thread i <- lane i)
// and waits for the load in the same asm statement, so no register is read early.
__device__ __forceinline__ void tmem_ld_x{n}(uint32_t taddr, uint32_t (&r)[{n}]) {{
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x{n}.b32 {{{outs}}}, [%{n}];\\n\\t"
      "tcgen05.wait::ld.sync.aligned;"
      : {cons}
      : "r"(taddr)
      : "memory");
}}
'''
def st(n):
    ins = ", ".join(f"%{i+1}" for i in range(n))
    cons = ", ".join(f'"r"(r[{i}])' for i in range(n))
    return f'''// Stores {n} consecutive 32-bit TMEM columns of this warp's 32 lanes (lane i <- thread i).
// Completion is awaited separately with tmem_wait_st().
__device__ __forceinline__ void tmem_st_x{n}(uint32_t taddr, const uint32_t (&r)[{n}]) {{
  asm volatile("tcgen05.st.sync.aligned.32x32b.x{n}.b32 [%0], {{{ins}}};"
               :
               : "r"(taddr), {cons}
               : "memory");
}}
'''
def ld_nowait(n):
    outs = ", ".join(f"%{i}" for i in range(n))
    cons = ", ".join(f'"=r"(r[{i}])' for i in range(n))
    return f'''// Starts loading {n} consecutive 32-bit TMEM columns (thread i <- lane i) without waiting:
// r must not be read before tmem_ld_wait_x{n}(r), which ties the registers to the wait.
__device__ __forceinline__ void tmem_ld_x{n}_async(uint32_t taddr, uint32_t (&r)[{n}]) {{
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x{n}.b32 {{{outs}}}, [%{n}];"
               : {cons}
               : "r"(taddr)
               : "memory");
}}
'''
def ld_wait(n):
    cons = ", ".join(f'"+r"(r[{i}])' for i in range(n))
    return f'''// Waits for this thread's outstanding TMEM loads; r (the destination of the load started
// by tmem_ld_x{n}_async) is an in-out operand, so no use of it moves above the wait.
__device__ __forceinline__ void tmem_ld_wait_x{n}(uint32_t (&r)[{n}]) {{
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : {cons}
               :
               : "memory");
}}
'''
hdr = '''// TMEM <-> register moves in the 32x32b shape: every thread of a warp owns one TMEM lane
// (one row of a 128-row accumulator) and a run of consecutive 32-bit columns.
// The operand lists are long but regular.
#pragma once
#include <cstdint>

namespace attn {

'''
body = (ld(16) + "\n" + ld(32) + "\n" + ld(64) + "\n" + ld(128) + "\n" + ld_nowait(32) + "\n" +
        ld_wait(32) + "\n" + ld_nowait(64) + "\n" + ld_wait(64) + "\n" + st(16) + "\n" + st(32))
open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tmem_ldst.cuh"), "w").write(hdr + body + "\n}  // namespace attn\n")
