"""Writes tmem_ldst.inc: inline-PTX wrappers for tcgen05.ld / tcgen05.st with the 32x32b shape (one TMEM lane
per thread, one 32-bit column per register), one function per register count, because an asm statement needs
its operands spelled out one by one.

    python exact_io_aware_76_b200/csrc/gen_tmem_ldst.py

  tmem_ld_xN(taddr, r)          N columns into r[0..N), then tcgen05.wait::ld (N = 16, 32, 64, 128)
  tmem_ld_xN_pair(a1, r1, a2, r2)  two N-column loads and one wait (N = 32, 64)
  tmem_st_xN(taddr, r)          N columns from r[0..N) (N = 16, 32, 64); the caller waits (tmem_st_wait)
"""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def _regs(first, n):
    return ",".join("%%%d" % (first + i) for i in range(n))


def ld(n):
    outs = ", ".join('"=r"(r[%d])' % i for i in range(n))
    return ('__device__ __forceinline__ void tmem_ld_x%d(uint32_t taddr, uint32_t* r) {\n'
            '  asm volatile("tcgen05.ld.sync.aligned.32x32b.x%d.b32 {%s}, [%%%d];\\n\\t"\n'
            '               "tcgen05.wait::ld.sync.aligned;"\n'
            '               : %s\n'
            '               : "r"(taddr) : "memory");\n'
            '}\n' % (n, n, _regs(0, n), n, outs))


def ld_pair(n):
    outs = ", ".join(['"=r"(r1[%d])' % i for i in range(n)] + ['"=r"(r2[%d])' % i for i in range(n)])
    return ('__device__ __forceinline__ void tmem_ld_x%d_pair(uint32_t a1, uint32_t* r1, uint32_t a2, uint32_t* r2) {\n'
            '  asm volatile("tcgen05.ld.sync.aligned.32x32b.x%d.b32 {%s}, [%%%d];\\n\\t"\n'
            '               "tcgen05.ld.sync.aligned.32x32b.x%d.b32 {%s}, [%%%d];\\n\\t"\n'
            '               "tcgen05.wait::ld.sync.aligned;"\n'
            '               : %s\n'
            '               : "r"(a1), "r"(a2) : "memory");\n'
            '}\n' % (n, n, _regs(0, n), 2 * n, n, _regs(n, n), 2 * n + 1, outs))


def st(n):
    ins = ", ".join('"r"(r[%d])' % i for i in range(n))
    return ('__device__ __forceinline__ void tmem_st_x%d(uint32_t taddr, const uint32_t* r) {\n'
            '  asm volatile("tcgen05.st.sync.aligned.32x32b.x%d.b32 [%%0], {%s};"\n'
            '               :: "r"(taddr), %s : "memory");\n'
            '}\n' % (n, n, _regs(1, n), ins))


def generate():
    out = ["// tmem_ldst.inc -- written by gen_tmem_ldst.py (do not edit by hand): tcgen05.ld (with its wait) and",
           "// tcgen05.st wrappers, shape 32x32b (lane = thread, one 32-bit column per register).", ""]
    out += [ld(n) for n in (16, 32, 64, 128)]
    out += [st(n) for n in (16, 32, 64)]
    out += ["// Two loads (e.g. the S^T and dP^T rows of one thread) and a single wait.", ld_pair(32), ld_pair(64)]
    return "\n".join(out)


if __name__ == "__main__":
    with open(os.path.join(HERE, "tmem_ldst.inc"), "w") as f:
        f.write(generate())
