"""Host-side checks of the C ABI (no GPU needed, no compute calls): the library loads and
exports every entry point include/dp.h declares, the ctypes mirrors match the C struct
layouts, and argument errors are reported synchronously before anything is enqueued."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dp.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:dp_status|const char\*|int32_t)\s+(dp_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def m():
    import long_video_diffusion_b200 as mod
    return mod


def test_library_exports_every_declared_function(m):
    declared = _declared_functions()
    assert len(declared) >= 13
    out = subprocess.run(["nm", "-D", "--defined-only", m.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dp_\w+)$", out, flags=re.M))
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    assert sorted(m.EXPORTS) == declared
    for f in declared:
        assert hasattr(m._lib, f)
    assert m.version() == 100


def test_status_strings(m):
    for code, name in [(0, "DP_OK"), (-1, "DP_ERR_INVALID_ARG"), (-5, "DP_ERR_TIMEOUT"), (-6, "DP_ERR_EMPTY")]:
        assert m._lib.dp_status_string(code).decode() == name


def test_ctypes_layouts_match_c(tmp_path, m):
    src = tmp_path / "layout.c"
    src.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "dp.h"
int main(void) {
  printf("%zu %zu %zu\\n", sizeof(dp_blocks), offsetof(dp_blocks, row_offset), offsetof(dp_blocks, mod));
  printf("%zu %zu %zu %zu\\n", sizeof(dp_kvcache), offsetof(dp_kvcache, len), offsetof(dp_kvcache, n_advances),
         offsetof(dp_kvcache, dtype));
  printf("%zu %zu %zu %zu\\n", sizeof(dp_queue), offsetof(dp_queue, rows), offsetof(dp_queue, n_pushed),
         offsetof(dp_queue, dtype));
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    b = [int(x) for x in lines[0].split()]
    c = [int(x) for x in lines[1].split()]
    q = [int(x) for x in lines[2].split()]
    assert b == [ctypes.sizeof(m.DpBlocks), m.DpBlocks.row_offset.offset, m.DpBlocks.mod.offset]
    assert c == [ctypes.sizeof(m.DpKvcache), m.DpKvcache.len.offset, m.DpKvcache.n_advances.offset,
                 m.DpKvcache.dtype.offset]
    assert q == [ctypes.sizeof(m.DpQueue), m.DpQueue.rows.offset, m.DpQueue.n_pushed.offset,
                 m.DpQueue.dtype.offset]


FAKE = 0x7f0000000000  # 16-byte aligned, never dereferenced: every call below fails its checks first


def _blocks(m, rows, hidden):
    b = m.DpBlocks()
    b.n_blocks = len(rows)
    b.hidden = hidden
    off = 0
    for i, r in enumerate(rows):
        b.row_offset[i] = off
        b.mod[i] = FAKE + 4096 * i
        off += r
    b.row_offset[len(rows)] = off
    return b


def test_blocks_from_table_checks(m):
    out = m.DpBlocks()
    ts = (ctypes.c_int32 * 2)(0, 1000)
    rows = (ctypes.c_int32 * 2)(4, 4)
    assert m._lib.dp_blocks_from_table(ctypes.byref(out), ctypes.c_void_p(FAKE), 1000, 64, ts, rows, 2) == m.ERR_INVALID_ARG
    ts = (ctypes.c_int32 * 2)(0, 999)
    assert m._lib.dp_blocks_from_table(ctypes.byref(out), ctypes.c_void_p(FAKE), 1000, 64, ts, rows, 2) == m.OK
    assert out.offsets == [0, 4, 8]
    assert out.mod[1] == FAKE + 999 * 3 * 64 * 4
    assert m._lib.dp_blocks_from_table(ctypes.byref(out), ctypes.c_void_p(FAKE), 1000, 64, ts, rows, 17) == m.ERR_INVALID_ARG


def _attn(m, q=FAKE, k=FAKE + 1024, v=FAKE + 2048, n=256, ck=FAKE + 4096, cv=FAKE + 8192, lc=128,
          out=FAKE + 16384, H=2, hd=64, blk=None, dt=1, ft=2):
    blk = blk if blk is not None else _blocks(m, [128, 128], H * hd)
    return m._lib.dp_window_attention(ctypes.c_void_p(q), ctypes.c_void_p(k), ctypes.c_void_p(v), n,
                                      ctypes.c_void_p(ck), ctypes.c_void_p(cv), lc, None, ctypes.c_void_p(out),
                                      H, hd, 0.0, ctypes.byref(blk), 3, dt, ft, None)


def test_attention_argument_errors(m):
    assert _attn(m, q=0) == m.ERR_INVALID_ARG                       # NULL
    assert _attn(m, q=FAKE + 8) == m.ERR_INVALID_ARG                # misaligned
    assert _attn(m, n=0, blk=_blocks(m, [0], 128)) == m.ERR_INVALID_ARG
    assert _attn(m, H=1, hd=96, blk=_blocks(m, [128, 128], 96)) == m.ERR_UNSUPPORTED
    assert _attn(m, H=1, hd=96, dt=0, ft=0, blk=_blocks(m, [128, 128], 96)) == m.ERR_UNSUPPORTED
    assert _attn(m, dt=0, ft=2) == m.ERR_UNSUPPORTED              # f32 window with f16 features
    assert _attn(m, dt=2, ft=2) == m.ERR_UNSUPPORTED              # f16 window
    assert _attn(m, blk=_blocks(m, [128, 127], 128)) == m.ERR_INVALID_ARG   # offsets != n_win
    assert _attn(m, out=FAKE) == m.ERR_INVALID_ARG                  # out aliases q
    assert _attn(m, lc=-1) == m.ERR_INVALID_ARG
    assert _attn(m, ck=0, lc=5) == m.ERR_INVALID_ARG
    bad = _blocks(m, [128, 128], 128)
    bad.mod[1] = 0
    assert _attn(m, blk=bad) == m.ERR_INVALID_ARG
    assert b"mod[1]" in m._lib.dp_last_error_detail()
    assert _attn(m, dt=7) == m.ERR_INVALID_ARG


def test_modulate_dtype_pairs(m):
    blk = _blocks(m, [8], 64)
    mod = lambda xd, yd: m._lib.dp_adaln_modulate(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + 4096), 8,
                                                  ctypes.byref(blk), xd, yd, None)
    assert mod(0, 2) == m.ERR_UNSUPPORTED        # f32 -> f16
    assert mod(2, 1) == m.ERR_UNSUPPORTED        # f16 -> bf16
    assert mod(1, 5) == m.ERR_INVALID_ARG


def _cache(m, capacity=128, hidden=128, n_slots=1, length=0, dt=2):
    c = m.DpKvcache()
    c.k, c.v = FAKE + (1 << 20), FAKE + (2 << 20)
    c.capacity, c.hidden, c.n_slots, c.dtype = capacity, hidden, n_slots, dt
    c.len[0] = length
    return c


def test_advance_capacity_errors(m):
    c = _cache(m)
    assert m._lib.dp_kvcache_advance(ctypes.byref(c), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), 129, None) == m.ERR_CAPACITY
    assert c.n_advances == 0
    c.len[0] = 200
    assert m._lib.dp_kvcache_advance(ctypes.byref(c), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), 1, None) == m.ERR_CAPACITY


def _queue(m, n_slots=2, slot_rows=64, hidden=128, count=0, rows=(), dt=1):
    q = m.DpQueue()
    q.latent = FAKE + (8 << 20)
    q.slot_rows, q.hidden, q.n_slots, q.count, q.dtype = slot_rows, hidden, n_slots, count, dt
    for i, r in enumerate(rows):
        q.rows[i] = r
    return q


def test_queue_host_logic(m):
    q = _queue(m)
    assert m._lib.dp_queue_pop(ctypes.byref(q)) == m.ERR_EMPTY
    full = _queue(m, count=2, rows=(64, 64))
    assert m._lib.dp_queue_push(ctypes.byref(full), ctypes.c_void_p(FAKE), 64, None) == m.ERR_CAPACITY
    short = _queue(m, n_slots=3, count=1, rows=(32,))
    assert m._lib.dp_queue_push(ctypes.byref(short), ctypes.c_void_p(FAKE), 64, None) == m.ERR_INVALID_ARG
    big = _queue(m, n_slots=3)
    assert m._lib.dp_queue_push(ctypes.byref(big), ctypes.c_void_p(FAKE), 65, None) == m.ERR_CAPACITY
    # pop is metadata only: head rotates, rows/evals shift toward the head
    q = _queue(m, n_slots=3, count=3, rows=(64, 64, 40))
    q.head = 2
    q.evals[0], q.evals[1], q.evals[2] = 9, 5, 1
    assert m._lib.dp_queue_pop(ctypes.byref(q)) == m.OK
    assert (q.head, q.count, q.n_popped) == (0, 2, 1)
    assert [q.rows[i] for i in range(2)] == [64, 40] and [q.evals[i] for i in range(2)] == [5, 1]


def test_queue_blocks_host_lookup(m):
    q = _queue(m, n_slots=4, slot_rows=64, count=3, rows=(64, 64, 16))
    q.head = 3
    q.evals[0], q.evals[1], q.evals[2] = 4, 2, 0
    tau = (ctypes.c_int32 * 5)(999, 750, 500, 250, 0)
    out = m.DpBlocks()
    win = ctypes.c_void_p()
    n = ctypes.c_int64()
    assert m._lib.dp_queue_blocks(ctypes.byref(q), ctypes.c_void_p(FAKE), 1000, tau, 5, ctypes.byref(out),
                                  ctypes.byref(win), ctypes.byref(n)) == m.OK
    assert n.value == 144 and out.offsets == [0, 64, 128, 144]
    assert win.value == FAKE + (8 << 20) + 3 * 64 * 128 * 2          # head slot of the mirrored ring
    assert [out.mod[i] for i in range(3)] == [FAKE + t * 3 * 128 * 4 for t in (0, 500, 999)]
    q.evals[0] = 5
    assert m._lib.dp_queue_blocks(ctypes.byref(q), ctypes.c_void_p(FAKE), 1000, tau, 5, ctypes.byref(out),
                                  ctypes.byref(win), ctypes.byref(n)) == m.ERR_INVALID_ARG


def test_window_step_checks_before_launch(m):
    blk = _blocks(m, [128, 128], 128)
    c = _cache(m, capacity=100)
    assert m._lib.dp_window_step(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), 256,
                                 ctypes.byref(blk), ctypes.byref(_cache(m, dt=1)), ctypes.c_void_p(FAKE + (64 << 20)),
                                 None, ctypes.c_void_p(FAKE + (32 << 20)), 2, 64, 0, None, None, 0, 1,
                                 None) == m.ERR_INVALID_ARG     # bf16 window needs an f16 feature cache
    args = lambda flags, queue=None, noise=None, rows=0: m._lib.dp_window_step(
        ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), 256, ctypes.byref(blk), ctypes.byref(c),
        ctypes.c_void_p(FAKE + (64 << 20)), None, ctypes.c_void_p(FAKE + (32 << 20)), 2, 64, flags,
        ctypes.byref(queue) if queue is not None else None, ctypes.c_void_p(noise) if noise else None, rows, 1, None)
    assert args(m.STEP_POP) == m.ERR_CAPACITY           # head block (128 rows) > cache capacity
    assert c.n_advances == 0
    c = _cache(m, capacity=128)
    assert args(0, noise=FAKE, rows=64) == m.ERR_INVALID_ARG        # push without a queue
    q = _queue(m, n_slots=2, slot_rows=128, count=2, rows=(128, 128))
    assert args(0, queue=q, noise=FAKE, rows=128) == m.ERR_CAPACITY  # full queue, no pop
    assert args(m.STEP_POP, queue=_queue(m, count=0)) == m.ERR_EMPTY


def test_sublayer_entry_points_check_before_launch(m):
    P = ctypes.c_void_p
    blk = _blocks(m, [128, 128], 256)
    lin = lambda a=FAKE, w=FAKE + 4096, n=256, k=256, y=FAKE + 8192, yd=1, mrows=256: m._lib.dp_linear(
        P(a), P(w), None, mrows, n, k, P(y), yd, None)
    assert lin(a=0) == m.ERR_INVALID_ARG
    assert lin(w=FAKE + 8) == m.ERR_INVALID_ARG                # misaligned
    assert lin(n=192) == m.ERR_UNSUPPORTED                      # n not a multiple of 128
    assert lin(k=100) == m.ERR_UNSUPPORTED                      # k not a multiple of 8
    assert lin(yd=0) == m.ERR_UNSUPPORTED                       # fp32 output
    assert lin(y=FAKE) == m.ERR_INVALID_ARG                     # y aliases a
    assert lin(mrows=0) == m.ERR_INVALID_ARG
    ln = lambda hidden=256, eps=1e-6, rows=(128, 128): m._lib.dp_ln_modulate(
        P(FAKE), P(FAKE + 4096), sum(rows), ctypes.byref(_blocks(m, list(rows), hidden)), eps, None)
    assert ln(hidden=128) == m.ERR_UNSUPPORTED                  # hidden not a multiple of 256
    assert ln(eps=0.0) == m.ERR_INVALID_ARG
    assert m._lib.dp_ln_modulate(P(FAKE), P(FAKE + 4096), 200, ctypes.byref(blk), 1e-6, None) == m.ERR_INVALID_ARG
    assert m._lib.dp_qkv_project(P(FAKE), P(FAKE + 4096), None, 256, 192, P(FAKE + 8192), P(FAKE + 16384),
                                 P(FAKE + 32768), None) == m.ERR_UNSUPPORTED
    assert m._lib.dp_qkv_project(P(FAKE), P(FAKE + 4096), None, 256, 256, P(FAKE), P(FAKE + 16384),
                                 P(FAKE + 32768), None) == m.ERR_INVALID_ARG      # q aliases h
    assert m._lib.dp_out_project(P(FAKE), P(FAKE + 4096), None, 256, ctypes.byref(blk), None, P(FAKE + 8192),
                                 None) == m.ERR_INVALID_ARG                          # no residual
    assert m._lib.dp_out_project(P(FAKE), P(FAKE + 4096), None, 256, ctypes.byref(blk), P(FAKE + 16384), P(FAKE),
                                 None) == m.ERR_INVALID_ARG                          # out aliases o
    c = _cache(m, capacity=100, hidden=256)
    step = lambda flags=0, x=FAKE, out=FAKE + (32 << 20), hd=64, queue=None: m._lib.dp_sublayer_step(
        P(x), 256, ctypes.byref(blk), P(FAKE + (8 << 20)), None, P(FAKE + (16 << 20)), None, 1e-6, ctypes.byref(c),
        P(FAKE + (64 << 20)), P(out), 256 // hd, hd, flags, ctypes.byref(queue) if queue is not None else None,
        None, 0, None)
    assert step(m.STEP_POP) == m.ERR_CAPACITY                  # head block (128 rows) > capacity 100
    assert c.n_advances == 0
    assert step(out=FAKE) == m.ERR_INVALID_ARG                  # out aliases x
    assert step(hd=32) == m.ERR_UNSUPPORTED                     # attention head_dim


def test_context_refresh_checks_before_launch(m):
    P = ctypes.c_void_p
    c = _cache(m, capacity=128, hidden=128, length=77)
    ref = lambda n=100, k=FAKE, v=FAKE + 65536, dt=1, rows=None, cache=c: m._lib.dp_context_refresh(
        P(k), P(v), n, ctypes.byref(_blocks(m, [n] if rows is None else rows, 128)), ctypes.byref(cache), dt, None)
    assert ref(dt=2) == m.ERR_UNSUPPORTED                        # f16 context rows
    assert ref(dt=0) == m.ERR_INVALID_ARG                        # f32 rows need an f32 cache
    assert ref(n=129) == m.ERR_CAPACITY                          # more rows than the slot holds
    assert ref(k=0) == m.ERR_INVALID_ARG
    assert ref(v=FAKE + 8) == m.ERR_INVALID_ARG                  # misaligned
    assert ref(k=FAKE + (1 << 20)) == m.ERR_INVALID_ARG          # rows inside the cache ring
    assert ref(rows=[50, 49]) == m.ERR_INVALID_ARG               # block table covers 99 of 100 rows
    assert c.len[0] == 77
    assert ref(n=0) == m.OK and c.len[0] == 0                    # empty context: nothing enqueued
    c2 = _cache(m, capacity=128, hidden=256, length=5)
    sub = lambda n=100, x=FAKE, work=FAKE + (4 << 20), eps=1e-6, hidden=256, cache=c2: \
        m._lib.dp_context_refresh_sublayer(P(x), n, ctypes.byref(_blocks(m, [n], hidden)), P(FAKE + (8 << 20)),
                                           None, eps, ctypes.byref(cache), P(work), None)
    assert sub(n=200) == m.ERR_CAPACITY
    assert sub(eps=0.0) == m.ERR_INVALID_ARG
    assert sub(hidden=128, cache=_cache(m, capacity=128, hidden=128)) == m.ERR_UNSUPPORTED
    assert sub(work=FAKE + 4096) == m.ERR_INVALID_ARG            # work overlaps x_ctx
    assert sub(work=FAKE + (2 << 20)) == m.ERR_INVALID_ARG       # work overlaps the cache ring
    assert sub(x=0) == m.ERR_INVALID_ARG
    assert c2.len[0] == 5
    assert sub(n=0) == m.OK and c2.len[0] == 0


def test_noalloc_scratch_size_and_capacity_checks(m):
    """The binding's NOALLOC_SCRATCH_BYTES is the header's DP_NOALLOC_SCRATCH_BYTES, and
    dp_window_step_noalloc rejects windows beyond it (absurd sizes included, whose byte count
    would overflow 64 bits) before it touches the GPU."""
    text = open(HEADER).read()
    mt = re.search(r"#define\s+DP_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert mt is not None
    assert m.NOALLOC_SCRATCH_BYTES == int(mt.group(1)) << int(mt.group(2))
    blk = _blocks(m, [128, 128], 128)
    cache = m.DpKvcache()

    def call(n, H, hd, dt):
        return m._lib.dp_window_step_noalloc(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE),
                                             n, ctypes.byref(blk), ctypes.byref(cache), None,
                                             ctypes.c_void_p(FAKE + 65536), H, hd, 0, None, None, 0, dt, None)

    cap = m.NOALLOC_SCRATCH_BYTES
    assert call(cap // (2 * 2048 * 2) + 1, 16, 128, m.BF16) == m.ERR_CAPACITY      # one bf16 row too many
    assert call(cap // (2 * 128 * 4) + 1, 2, 64, m.F32) == m.ERR_CAPACITY          # fp32 features: 4 bytes
    assert call(2 ** 62, 1 << 30, 1 << 30, m.BF16) == m.ERR_CAPACITY               # the product overflows
    assert call((1 << 62) + 1, 2, 64, m.BF16) == m.ERR_CAPACITY
    assert "scratch" in m._lib.dp_last_error_detail().decode()
    assert call(0, 2, 64, m.BF16) == m.ERR_INVALID_ARG
    assert cache.n_advances == 0
