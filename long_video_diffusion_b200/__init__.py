"""Python binding of the DualParal window-step library (libdp_b200.so, sm_100a).

Argument marshalling only: every step of the window step runs in the library's CUDA
kernels, and there is no fallback.  Importing fails loudly when the library has not been
built (``python long_video_diffusion_b200/_build.py``).  PyTorch supplies device memory,
streams and the current device; tensors are passed as raw pointers.

The calls mirror include/dp.h:
  blocks_from_table, queue_blocks   A0  per-block adaLN lookup (host)
  adaln_modulate                    A1  modulation prepass
  window_attention                  A2  attention over [cache ; window], fused Q prologue
                                        and gate (+ residual) epilogue
  kvcache_advance, queue_push/pop   A3  queue and cache advance
  window_step                       A4  the whole step
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdp_b200.so")

MAX_BLOCKS = 16
MAX_SLOTS = 16

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_CAPACITY, ERR_TIMEOUT, ERR_EMPTY = 0, -1, -2, -3, -4, -5, -6
F32, BF16, F16 = 0, 1, 2
MOD_Q, GATE_OUT = 1, 2
TEST_SKIP_KV_LOADS = 0x80000000
STEP_POP = 1
STEP_CACHE_ALL_SLOTS = 2

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python long_video_diffusion_b200/_build.py` "
                      "(nvcc, sm_100a). There is no non-CUDA implementation.")
_lib = ctypes.CDLL(LIB_PATH)


class DpBlocks(ctypes.Structure):
    _fields_ = [("n_blocks", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("row_offset", ctypes.c_int32 * (MAX_BLOCKS + 1)),
                ("mod", ctypes.c_void_p * MAX_BLOCKS)]

    @property
    def offsets(self):
        return [self.row_offset[i] for i in range(self.n_blocks + 1)]


class DpKvcache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("capacity", ctypes.c_int64),
                ("hidden", ctypes.c_int32), ("n_slots", ctypes.c_int32),
                ("len", ctypes.c_int64 * MAX_SLOTS), ("n_advances", ctypes.c_int64),
                ("dtype", ctypes.c_int32)]


class DpQueue(ctypes.Structure):
    _fields_ = [("latent", ctypes.c_void_p), ("slot_rows", ctypes.c_int64), ("hidden", ctypes.c_int32),
                ("n_slots", ctypes.c_int32), ("head", ctypes.c_int32), ("count", ctypes.c_int32),
                ("rows", ctypes.c_int32 * MAX_SLOTS), ("evals", ctypes.c_int32 * MAX_SLOTS),
                ("n_pushed", ctypes.c_int64), ("n_popped", ctypes.c_int64), ("dtype", ctypes.c_int32)]


class DpFifo(ctypes.Structure):
    _fields_ = [("n_blocks", ctypes.c_int32), ("n_timesteps", ctypes.c_int32), ("window_blocks", ctypes.c_int32),
                ("next_block", ctypes.c_int32), ("step", ctypes.c_int64), ("exited_rows", ctypes.c_int64)]


class DpFifoStep(ctypes.Structure):
    _fields_ = [("push_before", ctypes.c_int32), ("pop", ctypes.c_int32), ("push_after", ctypes.c_int32),
                ("done", ctypes.c_int32), ("exit_rows", ctypes.c_int64), ("ctx_rows", ctypes.c_void_p),
                ("ctx_n", ctypes.c_int64)]


_P = ctypes.c_void_p
_I32, _I64, _U32, _F = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float
_SIGS = {
    "dp_blocks_from_table": [ctypes.POINTER(DpBlocks), _P, _I32, _I32, ctypes.POINTER(_I32),
                             ctypes.POINTER(_I32), _I32],
    "dp_queue_blocks": [ctypes.POINTER(DpQueue), _P, _I32, ctypes.POINTER(_I32), _I32,
                        ctypes.POINTER(DpBlocks), ctypes.POINTER(_P), ctypes.POINTER(_I64)],
    "dp_adaln_modulate": [_P, _P, _I64, ctypes.POINTER(DpBlocks), _I32, _I32, _P],
    "dp_window_attention": [_P, _P, _P, _I64, _P, _P, _I64, _P, _P, _I32, _I32, _F,
                            ctypes.POINTER(DpBlocks), _U32, _I32, _I32, _P],
    "dp_kvcache_advance": [ctypes.POINTER(DpKvcache), _P, _P, _I64, _P],
    "dp_queue_push": [ctypes.POINTER(DpQueue), _P, _I64, _P],
    "dp_queue_pop": [ctypes.POINTER(DpQueue)],
    "dp_queue_push_frames": [ctypes.POINTER(DpQueue), _P, _I32, _I64, ctypes.POINTER(_I32), _I32, _P],
    "dp_fifo_entry_step": [_I32, _I32, _I32, ctypes.POINTER(_I64)],
    "dp_fifo_init": [ctypes.POINTER(DpFifo), _I32, _I32, _I32],
    "dp_fifo_plan": [ctypes.POINTER(DpFifo), ctypes.POINTER(DpQueue), ctypes.POINTER(DpFifoStep)],
    "dp_fifo_commit": [ctypes.POINTER(DpFifo), ctypes.POINTER(DpFifoStep)],
    "dp_coordinated_frames": [ctypes.POINTER(_I32), _I32, _I32, _I32, ctypes.POINTER(_I32), _I32,
                              ctypes.POINTER(_I32), ctypes.POINTER(_I32)],
    "dp_window_step": [_P, _P, _P, _I64, ctypes.POINTER(DpBlocks), ctypes.POINTER(DpKvcache), _P, _P, _P,
                       _I32, _I32, _U32, ctypes.POINTER(DpQueue), _P, _I64, _I32, _P],
    "dp_window_step_noalloc": [_P, _P, _P, _I64, ctypes.POINTER(DpBlocks), ctypes.POINTER(DpKvcache), _P, _P,
                               _I32, _I32, _U32, ctypes.POINTER(DpQueue), _P, _I64, _I32, _P],
    "dp_ln_modulate": [_P, _P, _I64, ctypes.POINTER(DpBlocks), _F, _P],
    "dp_linear": [_P, _P, _P, _I64, _I32, _I32, _P, _I32, _P],
    "dp_qkv_project": [_P, _P, _P, _I64, _I32, _P, _P, _P, _P],
    "dp_out_project": [_P, _P, _P, _I64, ctypes.POINTER(DpBlocks), _P, _P, _P],
    "dp_sublayer_step": [_P, _I64, ctypes.POINTER(DpBlocks), _P, _P, _P, _P, _F, ctypes.POINTER(DpKvcache), _P, _P,
                         _I32, _I32, _U32, ctypes.POINTER(DpQueue), _P, _I64, _P],
    "dp_context_refresh": [_P, _P, _I64, ctypes.POINTER(DpBlocks), ctypes.POINTER(DpKvcache), _I32, _P],
    "dp_context_refresh_sublayer": [_P, _I64, ctypes.POINTER(DpBlocks), _P, _P, _F, ctypes.POINTER(DpKvcache), _P,
                                    _P],
    "dp_profile_begin": [_I32],
    "dp_profile_end": [ctypes.POINTER(_F), ctypes.POINTER(_F), ctypes.POINTER(_F), ctypes.POINTER(_I32)],
    "dp_profile_end_stages": [ctypes.POINTER(_F), _I32, ctypes.POINTER(_I32), ctypes.POINTER(_I32)],
    "dp_set_device": [_I32],
    "dp_device_status": [_P],
    "dp_status_string": [_I32],
    "dp_last_error_detail": [],
    "dp_version": [],
}
for _name, _args in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int32
_lib.dp_status_string.restype = ctypes.c_char_p
_lib.dp_last_error_detail.restype = ctypes.c_char_p

EXPORTS = sorted(_SIGS)


class DpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = _lib.dp_last_error_detail().decode(errors="replace")
        name = _lib.dp_status_string(status).decode()
        super().__init__(f"{where}: {name} ({detail})")


def _check(status: int, where: str) -> None:
    if status != OK:
        raise DpError(status, where)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.float16:
        return F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor, stream=None):
    dev = t.device.index if t.device.index is not None else torch.cuda.current_device()
    _check(_lib.dp_set_device(dev), "dp_set_device")
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    return ctypes.c_void_p(s.cuda_stream)


def version() -> int:
    return _lib.dp_version()


# ------------------------------------------------------------------------- A0

def blocks_from_table(table: torch.Tensor, timesteps: Sequence[int], block_rows: Sequence[int]) -> DpBlocks:
    """Block table whose block b uses rows block_rows[b] and adaLN row table[timesteps[b]]."""
    if table.dtype != torch.float32 or table.dim() != 3 or table.shape[1] != 3:
        raise ValueError("table must be float32 [T, 3, hidden]")
    n = len(timesteps)
    if len(block_rows) != n:
        raise ValueError("timesteps and block_rows differ in length")
    out = DpBlocks()
    ts = (ctypes.c_int32 * max(n, 1))(*timesteps)
    rows = (ctypes.c_int32 * max(n, 1))(*block_rows)
    _check(_lib.dp_blocks_from_table(ctypes.byref(out), _ptr(table), table.shape[0], table.shape[2], ts, rows, n),
           "dp_blocks_from_table")
    out._table = table  # keep the table alive while the block table is in use
    return out


# ------------------------------------------------------------------------- state

def feature_dtype(window_dtype: torch.dtype) -> torch.dtype:
    """Element type of the modulated features k', v' and of the cache for a window of
    ``window_dtype``: f16 for bf16 windows, f32 for f32 windows."""
    return torch.float32 if window_dtype == torch.float32 else torch.float16


class KVCache:
    """The feature-cache ring (device buffers [n_slots, capacity, hidden] owned here)."""

    def __init__(self, capacity: int, hidden: int, dtype=torch.float16, n_slots: int = 1,
                 device="cuda", k: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None,
                 length: int = 0):
        self.k = torch.zeros(n_slots, capacity, hidden, dtype=dtype, device=device) if k is None else k
        self.v = torch.zeros(n_slots, capacity, hidden, dtype=dtype, device=device) if v is None else v
        if self.k.shape != (n_slots, capacity, hidden) or self.v.shape != self.k.shape:
            raise ValueError("cache buffers must be [n_slots, capacity, hidden]")
        self.desc = DpKvcache()
        self.desc.k = self.k.data_ptr()
        self.desc.v = self.v.data_ptr()
        self.desc.capacity = capacity
        self.desc.hidden = hidden
        self.desc.n_slots = n_slots
        self.desc.len[0] = length
        self.desc.n_advances = 0
        self.desc.dtype = _dtype(self.k)

    @property
    def n_advances(self) -> int:
        return self.desc.n_advances

    def read_slot(self) -> int:
        d = self.desc
        return (d.n_advances - 1) % d.n_slots if d.n_advances > 0 else 0

    @property
    def length(self) -> int:
        return self.desc.len[self.read_slot()]


class Queue:
    """The latent block queue: a mirrored ring [2 * n_slots, slot_rows, hidden] owned here."""

    def __init__(self, n_slots: int, slot_rows: int, hidden: int, dtype=torch.bfloat16, device="cuda"):
        self.latent = torch.zeros(2 * n_slots, slot_rows, hidden, dtype=dtype, device=device)
        self.desc = DpQueue()
        self.desc.latent = self.latent.data_ptr()
        self.desc.slot_rows = slot_rows
        self.desc.hidden = hidden
        self.desc.n_slots = n_slots
        self.desc.head = 0
        self.desc.count = 0
        self.desc.dtype = _dtype(self.latent)

    @property
    def count(self) -> int:
        return self.desc.count

    @property
    def head(self) -> int:
        return self.desc.head

    def rows(self):
        return [self.desc.rows[i] for i in range(self.desc.count)]

    def evals(self):
        return [self.desc.evals[i] for i in range(self.desc.count)]

    def window_rows(self) -> int:
        return sum(self.rows())

    def window(self) -> torch.Tensor:
        """View of the live window (head block first) inside the mirrored ring."""
        flat = self.latent.view(-1, self.desc.hidden)
        start = self.desc.head * self.desc.slot_rows
        return flat[start:start + self.window_rows()]


def queue_blocks(queue: Queue, table: torch.Tensor, tau: Sequence[int]):
    """(block table, window pointer, n_win) of the queue's live window."""
    out = DpBlocks()
    tarr = (ctypes.c_int32 * len(tau))(*tau)
    win = ctypes.c_void_p()
    n = ctypes.c_int64()
    _check(_lib.dp_queue_blocks(ctypes.byref(queue.desc), _ptr(table), table.shape[0], tarr, len(tau),
                                ctypes.byref(out), ctypes.byref(win), ctypes.byref(n)), "dp_queue_blocks")
    out._table = table
    return out, win.value, n.value


# ------------------------------------------------------------------------- A1..A4

def adaln_modulate(x: torch.Tensor, y: torch.Tensor, blocks: DpBlocks, stream=None) -> None:
    """y = x * (1 + scale_b) + shift_b, rounded to y's dtype (bf16->bf16, bf16->f16, f16->f16, f32->f32)."""
    _check(_lib.dp_adaln_modulate(_ptr(x), _ptr(y), x.shape[0], ctypes.byref(blocks), _dtype(x), _dtype(y),
                                  _stream(x, stream)), "dp_adaln_modulate")


def window_attention(q, k, v, cache_k, cache_v, cache_len: int, out, n_heads: int, head_dim: int,
                     blocks: DpBlocks, flags: int = MOD_Q | GATE_OUT, residual=None,
                     softmax_scale: float = 0.0, stream=None) -> None:
    _check(_lib.dp_window_attention(_ptr(q), _ptr(k), _ptr(v), q.shape[0], _ptr(cache_k), _ptr(cache_v),
                                    int(cache_len), _ptr(residual), _ptr(out), n_heads, head_dim,
                                    float(softmax_scale), ctypes.byref(blocks), flags, _dtype(q), _dtype(k),
                                    _stream(q, stream)), "dp_window_attention")


def kvcache_advance(cache: KVCache, k_exit: torch.Tensor, v_exit: torch.Tensor, n_exit: int, stream=None) -> None:
    _check(_lib.dp_kvcache_advance(ctypes.byref(cache.desc), _ptr(k_exit), _ptr(v_exit), int(n_exit),
                                   _stream(cache.k, stream)), "dp_kvcache_advance")


def queue_push(queue: Queue, noise: torch.Tensor, rows: Optional[int] = None, stream=None) -> None:
    r = noise.shape[0] if rows is None else rows
    _check(_lib.dp_queue_push(ctypes.byref(queue.desc), _ptr(noise), int(r), _stream(queue.latent, stream)),
           "dp_queue_push")


def queue_push_frames(queue: Queue, pool: torch.Tensor, frames: Sequence[int], stream=None) -> None:
    """Push a block made of pool frames (dp_queue_push_frames); pool [frames][frame_rows][hidden]."""
    idx = (_I32 * len(frames))(*[int(f) for f in frames])
    _check(_lib.dp_queue_push_frames(ctypes.byref(queue.desc), _ptr(pool), pool.shape[0], pool.shape[1], idx,
                                     len(frames), _stream(queue.latent, stream)), "dp_queue_push_frames")


def coordinated_frames(block_frames: Sequence[int], window_blocks: int, b: int, prev_frames: Sequence[int],
                       perm: Optional[Sequence[int]]) -> list:
    """Pool frames of block b under the coordinated noise initialisation
    (dp_coordinated_frames): the pool is the first window's frames; block b < window_blocks
    takes its own frames in order, a later block the pool's frames in the order of the random
    permutation perm without prev_frames (the block before it)."""
    n = len(block_frames)
    bf = (_I32 * n)(*[int(f) for f in block_frames])
    prev = (_I32 * max(1, len(prev_frames)))(*[int(f) for f in prev_frames])
    pm = None if perm is None else (_I32 * len(perm))(*[int(f) for f in perm])
    nf = int(block_frames[b]) if 0 <= b < n else 1
    out = (_I32 * max(1, nf))()
    _check(_lib.dp_coordinated_frames(bf, n, int(window_blocks), int(b), prev, len(prev_frames), pm, out),
           "dp_coordinated_frames")
    return [out[i] for i in range(nf)]


def coordinated_schedule(block_frames: Sequence[int], window_blocks: int, perms) -> list:
    """Pool frames of every block of a video, block b from perms[b] (dp_coordinated_frames
    block after block)."""
    lists: list = []
    for b in range(len(block_frames)):
        lists.append(coordinated_frames(block_frames, window_blocks, b, lists[b - 1] if b else [],
                                        perms[b] if b >= window_blocks else None))
    return lists


def queue_pop(queue: Queue) -> None:
    _check(_lib.dp_queue_pop(ctypes.byref(queue.desc)), "dp_queue_pop")


def window_step(q, k, v, blocks: DpBlocks, cache: KVCache, kv_work, out, n_heads: int, head_dim: int,
                pop: bool = False, queue: Optional[Queue] = None, push_noise=None, push_rows=None,
                residual=None, stream=None, n_win: Optional[int] = None, cache_all_slots: bool = False) -> None:
    """One window step (see dp_window_step).  q, k, v are tensors or raw device addresses
    (n_win then required), e.g. the queue's live window.  kv_work holds at least
    2 * n_win * hidden feature elements (k' first, v' at element n_win * hidden).
    cache_all_slots: attend to every cache slot that holds rows (DP_STEP_CACHE_ALL_SLOTS)."""
    if isinstance(q, torch.Tensor):
        ref = q
        n = q.shape[0]
        qp, kp, vp = _ptr(q), _ptr(k), _ptr(v)
    else:
        ref = out
        n = int(n_win)
        qp, kp, vp = ctypes.c_void_p(q), ctypes.c_void_p(k), ctypes.c_void_p(v)
    rows = 0 if push_noise is None else (push_noise.shape[0] if push_rows is None else push_rows)
    _check(_lib.dp_window_step(qp, kp, vp, n, ctypes.byref(blocks), ctypes.byref(cache.desc), _ptr(kv_work),
                               _ptr(residual), _ptr(out), n_heads, head_dim,
                               (STEP_POP if pop else 0) | (STEP_CACHE_ALL_SLOTS if cache_all_slots else 0),
                               ctypes.byref(queue.desc) if queue is not None else None, _ptr(push_noise),
                               int(rows), _dtype(out), _stream(ref, stream)), "dp_window_step")


# ------------------------------------------------------------------------- host-fed steps

class StepPipeline:
    """Steps fed from host memory with the copies overlapped with the compute.

    Step i's inputs (pinned host tensors) are copied on a copy stream into one of ``depth``
    device buffer sets while step i - 1 computes on the compute stream, and step i - 1's
    output is read back on a third stream while step i computes.  Events order the three: a
    buffer set is refilled only after the step that used it has finished computing, and the
    output buffer only after its read-back.  Queue and cache descriptors advance in
    submission order as usual.  finish() waits for everything submitted.

    shapes: the device shapes of the step's inputs, in the order submit_with() receives them
    (for submit(): q, k, v and the noise block); out_shape: the step's output."""

    def __init__(self, n_win: int, hidden: int, noise_rows: int, dtype=torch.bfloat16, depth: int = 2,
                 device=None, shapes=None, out_shape=None):
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.depth = depth
        if shapes is None:
            shapes = [(n_win, hidden)] * 3 + [(noise_rows, hidden)]
        out_shape = out_shape or (n_win, hidden)
        self.inputs = [[torch.empty(*sh, dtype=dtype, device=dev) for sh in shapes] for _ in range(depth)]
        self.out = [torch.empty(*out_shape, dtype=dtype, device=dev) for _ in range(depth)]
        self.h2d = torch.cuda.Stream(dev)
        self.compute = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event() for _ in range(depth)]
        self.copied, self.computed, self.read = ev(), ev(), ev()
        self.n = 0

    def submit_with(self, host_inputs, hout, run) -> None:
        """Enqueue one step: copy host_inputs (pinned; None entries are skipped) into a device
        buffer set, call run(device_inputs, device_out, compute_stream) to enqueue the step's
        work, and read device_out back into hout."""
        i = self.n % self.depth
        dins = self.inputs[i]
        with torch.cuda.stream(self.h2d):
            if self.n >= self.depth:
                self.h2d.wait_event(self.computed[i])      # the step that used buffer set i is done
            for d, h in zip(dins, host_inputs):
                if h is not None:
                    d[:h.shape[0]].copy_(h, non_blocking=True)
            self.copied[i].record(self.h2d)
        self.compute.wait_event(self.copied[i])
        if self.n >= self.depth:
            self.compute.wait_event(self.read[i])          # out[i] has been read back
        run(dins, self.out[i], self.compute)
        self.computed[i].record(self.compute)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.computed[i])
            hout.copy_(self.out[i][:hout.shape[0]], non_blocking=True)
            self.read[i].record(self.d2h)
        self.n += 1

    def submit(self, hq, hk, hv, hnoise, hout, blocks: DpBlocks, cache: KVCache, kv_work, n_heads: int,
               head_dim: int, pop: bool = True, queue: Optional[Queue] = None) -> None:
        """One window step (dp_window_step) on host inputs hq, hk, hv, hnoise (pinned; hnoise may
        be None), its output read back into hout."""
        rows = None if hnoise is None else hnoise.shape[0]

        def run(d, out, stream):
            window_step(d[0], d[1], d[2], blocks, cache, kv_work, out, n_heads, head_dim, pop=pop, queue=queue,
                        push_noise=None if rows is None else d[3][:rows], stream=stream)
        self.submit_with([hq, hk, hv, hnoise], hout, run)

    def finish(self) -> None:
        for s in (self.h2d, self.compute, self.d2h):
            s.synchronize()


# ------------------------------------------------------------------------- B: DiT attention sublayer

LN_EPS = 1e-6


def ln_modulate(x, h, blocks: DpBlocks, eps: float = LN_EPS, stream=None) -> None:
    """h = LN(x) * (1 + scale_b) + shift_b (dp_ln_modulate); x, h bf16 [rows][hidden]."""
    _check(_lib.dp_ln_modulate(_ptr(x), _ptr(h), x.shape[0], ctypes.byref(blocks), float(eps), _stream(x, stream)),
           "dp_ln_modulate")


def linear(a, w, bias, y, stream=None) -> None:
    """y = a W^T + bias on the tensor cores (dp_linear); a [m][k] and w [n][k] bf16, bias
    float [n] or None, y bf16 or f16 [m][n]."""
    _check(_lib.dp_linear(_ptr(a), _ptr(w), _ptr(bias), a.shape[0], w.shape[0], a.shape[1], _ptr(y), _dtype(y),
                          _stream(a, stream)), "dp_linear")


def qkv_project(h, w_qkv, b_qkv, q, k, v, stream=None) -> None:
    """[q | k | v] = h W_qkv^T + b_qkv (dp_qkv_project): q bf16, k and v f16."""
    _check(_lib.dp_qkv_project(_ptr(h), _ptr(w_qkv), _ptr(b_qkv), h.shape[0], h.shape[1], _ptr(q), _ptr(k), _ptr(v),
                               _stream(h, stream)), "dp_qkv_project")


def out_project(o, w_o, b_o, blocks: DpBlocks, residual, out, stream=None) -> None:
    """out = residual + gate_b * (o W_o^T + b_o) (dp_out_project), bf16."""
    _check(_lib.dp_out_project(_ptr(o), _ptr(w_o), _ptr(b_o), o.shape[0], ctypes.byref(blocks), _ptr(residual),
                               _ptr(out), _stream(o, stream)), "dp_out_project")


def sublayer_work(n_win: int, hidden: int, device=None) -> torch.Tensor:
    """Scratch for sublayer_step: h / attention output, q, k, v (16-bit, n_win x hidden each)."""
    return torch.empty(4 * n_win * hidden, dtype=torch.bfloat16, device=device or "cuda")


def sublayer_step(x, blocks: DpBlocks, w_qkv, b_qkv, w_o, b_o, cache: KVCache, work, out, n_heads: int,
                  head_dim: int, eps: float = LN_EPS, pop: bool = False, queue: Optional[Queue] = None,
                  push_noise=None, push_rows=None, stream=None, n_win: Optional[int] = None,
                  cache_all_slots: bool = False) -> None:
    """One DiT attention-sublayer step (dp_sublayer_step).  x is a tensor or a raw device
    address (n_win then required), e.g. the queue's live window; work from sublayer_work.
    After the call, work's planes 2 and 3 hold the window's projected k and v (f16)."""
    if isinstance(x, torch.Tensor):
        ref, n, xp = x, x.shape[0], _ptr(x)
    else:
        ref, n, xp = out, int(n_win), ctypes.c_void_p(x)
    rows = 0 if push_noise is None else (push_noise.shape[0] if push_rows is None else push_rows)
    _check(_lib.dp_sublayer_step(xp, n, ctypes.byref(blocks), _ptr(w_qkv), _ptr(b_qkv), _ptr(w_o), _ptr(b_o),
                                 float(eps), ctypes.byref(cache.desc), _ptr(work), _ptr(out), n_heads, head_dim,
                                 (STEP_POP if pop else 0) | (STEP_CACHE_ALL_SLOTS if cache_all_slots else 0),
                                 ctypes.byref(queue.desc) if queue is not None else None,
                                 _ptr(push_noise), int(rows), _stream(ref, stream)), "dp_sublayer_step")


# ------------------------------------------------------------------------- C: fresh context

def context_refresh(k_ctx, v_ctx, ctx_blocks: DpBlocks, cache: KVCache, stream=None) -> None:
    """Recompute the context K/V of the window step now (dp_context_refresh): k' = k_ctx *
    (1 + scale_b) + shift_b, v' likewise, written over the cache slot the next step reads;
    k_ctx, v_ctx [n_ctx][hidden] bf16 (f16 cache) or f32 (f32 cache)."""
    if v_ctx.shape != k_ctx.shape or v_ctx.dtype != k_ctx.dtype:
        raise ValueError("k_ctx and v_ctx differ in shape or dtype")
    _check(_lib.dp_context_refresh(_ptr(k_ctx), _ptr(v_ctx), k_ctx.shape[0], ctypes.byref(ctx_blocks),
                                   ctypes.byref(cache.desc), _dtype(k_ctx), _stream(k_ctx, stream)),
           "dp_context_refresh")


def context_refresh_sublayer(x_ctx, ctx_blocks: DpBlocks, w_qkv, b_qkv, cache: KVCache, work,
                             eps: float = LN_EPS, stream=None) -> None:
    """Recompute the context K/V of the sublayer now (dp_context_refresh_sublayer): pre-norm
    with the context block's adaLN vectors, then the k and v thirds of the q/k/v projection,
    written over the cache slot the next step reads; x_ctx [n_ctx][hidden] bf16, work at
    least n_ctx * hidden bf16 elements (e.g. sublayer_work's first plane)."""
    if work.numel() * work.element_size() < x_ctx.numel() * 2:
        raise ValueError("work holds fewer than n_ctx * hidden 16-bit elements")
    _check(_lib.dp_context_refresh_sublayer(_ptr(x_ctx), x_ctx.shape[0], ctypes.byref(ctx_blocks), _ptr(w_qkv),
                                            _ptr(b_qkv), float(eps), ctypes.byref(cache.desc), _ptr(work),
                                            _stream(x_ctx, stream)), "dp_context_refresh_sublayer")


def sublayer_planes(work, n_win: int, hidden: int):
    """Views of the sublayer scratch: (o, q, k, v), each [n_win][hidden]."""
    plane = n_win * hidden
    o = work[:plane].view(n_win, hidden)
    q = work[plane:2 * plane].view(n_win, hidden)
    k = work[2 * plane:3 * plane].view(torch.float16).view(n_win, hidden)
    v = work[3 * plane:4 * plane].view(torch.float16).view(n_win, hidden)
    return o, q, k, v


def profile_begin(max_steps: int) -> None:
    """Time the stages of the next max_steps window_step calls on this thread."""
    _check(_lib.dp_profile_begin(int(max_steps)), "dp_profile_begin")


def profile_end():
    """(ms_modulate, ms_attention, ms_advance, steps): summed stage times since profile_begin."""
    a, b, c = ctypes.c_float(), ctypes.c_float(), ctypes.c_float()
    n = ctypes.c_int32()
    _check(_lib.dp_profile_end(ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), ctypes.byref(n)),
           "dp_profile_end")
    return a.value, b.value, c.value, n.value


def profile_end_stages(max_stages: int = 5):
    """([ms per stage], n_stages, steps) summed since profile_begin (dp_profile_end_stages):
    window steps 0 modulation, 1 attention, 2 advance; sublayer steps 0 pre-norm, 1 q/k/v
    projection, 2 attention, 3 out projection, 4 advance."""
    ms = (_F * max_stages)()
    ns, n = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.dp_profile_end_stages(ms, max_stages, ctypes.byref(ns), ctypes.byref(n)), "dp_profile_end_stages")
    return [ms[i] for i in range(max_stages)], ns.value, n.value


NOALLOC_SCRATCH_BYTES = 32 << 20   # DP_NOALLOC_SCRATCH_BYTES of include/dp.h (a CPU test keeps them equal)


def window_step_noalloc(q, k, v, blocks: DpBlocks, cache: KVCache, out, n_heads: int, head_dim: int,
                        pop: bool = False, queue: Optional[Queue] = None, push_noise=None, push_rows=None,
                        residual=None, stream=None, n_win: Optional[int] = None,
                        cache_all_slots: bool = False) -> None:
    """window_step without kv_work, for callers that cannot allocate device memory: the
    k'/v' scratch is a fixed NOALLOC_SCRATCH_BYTES array inside the library (see
    dp_window_step_noalloc).  Calls share that array, so they must not overlap on the GPU."""
    if isinstance(q, torch.Tensor):
        ref = q
        n = q.shape[0]
        qp, kp, vp = _ptr(q), _ptr(k), _ptr(v)
    else:
        ref = out
        n = int(n_win)
        qp, kp, vp = ctypes.c_void_p(q), ctypes.c_void_p(k), ctypes.c_void_p(v)
    rows = 0 if push_noise is None else (push_noise.shape[0] if push_rows is None else push_rows)
    _check(_lib.dp_window_step_noalloc(qp, kp, vp, n, ctypes.byref(blocks), ctypes.byref(cache.desc),
                                       _ptr(residual), _ptr(out), n_heads, head_dim,
                                       (STEP_POP if pop else 0) | (STEP_CACHE_ALL_SLOTS if cache_all_slots else 0),
                                       ctypes.byref(queue.desc) if queue is not None else None,
                                       _ptr(push_noise), int(rows), _dtype(out), _stream(ref, stream)),
           "dp_window_step_noalloc")


def device_status(stream=None) -> int:
    """Synchronize and read/clear the device status word; raises DpError on a timeout."""
    s = stream if stream is not None else torch.cuda.current_stream()
    st = _lib.dp_device_status(ctypes.c_void_p(s.cuda_stream))
    _check(st, "dp_device_status")
    return st


def loaded_library_path() -> str:
    return LIB_PATH


# ------------------------------------------------------------------------- long-video run

def fifo_entry_step(b: int, n_timesteps: int, window_blocks: int) -> int:
    """Step at which block b enters the queue (dp_fifo_entry_step)."""
    out = _I64()
    _check(_lib.dp_fifo_entry_step(int(b), int(n_timesteps), int(window_blocks), ctypes.byref(out)),
           "dp_fifo_entry_step")
    return out.value


def run_fifo(noise_blocks, table: torch.Tensor, tau: Sequence[int], window_blocks: int, cache: KVCache,
             queue: Queue, kv_work: torch.Tensor, out: torch.Tensor, n_heads: int, head_dim: int,
             on_step=None, stream=None, max_steps: Optional[int] = None, cache_all_slots: bool = False,
             frame_pool=None, fresh_t: Optional[int] = None, state: Optional["FifoState"] = None) -> int:
    """Denoise a whole video through the block queue (the pages' FIFO: push a noisy block at
    the tail, pop a clean block at the head; every block is evaluated once per step at its
    own timestep tau[evals]).  The schedule (which block enters when, when the head exits)
    is the library's (dp_fifo_plan / dp_fifo_commit); this loop only carries out its steps.
    q = k = v = the queue's live window (identity projections).  noise_blocks: device
    tensors in entry order.  out: one output tensor, or a list that the steps use in turn
    (step s writes out[s % len(out)], e.g. so that a step's output can be read back while
    the next step runs).  on_step(step, n_win, popped, pushed) is called after each step is
    enqueued.  max_steps stops the run early (the queue and cache are then left mid-run).
    cache_all_slots: every step attends to all of the cache ring's slots (the last n_slots
    exited blocks).  frame_pool = (pool, frame_lists): blocks are pushed as pool frames
    (dp_queue_push_frames; the coordinated noise initialisation) and noise_blocks only gives
    each block's row count.  fresh_t: before every step after the first exit, the context
    K/V are recomputed (dp_context_refresh) from the latent rows of the block that left last,
    conditioned on table[fresh_t], instead of reused from its last evaluation; the queue
    keeps those rows in the slot behind its head, so it needs more slots than
    window_blocks.  state: the run's progress (FifoState), updated as steps are enqueued; a
    run stopped by max_steps continues from it, also after checkpoint/restore.  Returns the
    number of steps run so far (state.step)."""
    T = len(tau)
    n_blocks = len(noise_blocks)
    if fresh_t is not None and queue.desc.n_slots <= window_blocks:
        raise ValueError("a fresh context needs a queue with more slots than window blocks")
    st = state if state is not None else FifoState()
    st.bind(n_blocks, T, window_blocks)
    plan = DpFifoStep()
    lat = queue.latent

    def push_block(b):
        if frame_pool is None:
            queue_push(queue, noise_blocks[b], stream=stream)
        else:
            queue_push_frames(queue, frame_pool[0], frame_pool[1][b], stream=stream)

    run = 0
    while max_steps is None or run < max_steps:
        _check(_lib.dp_fifo_plan(ctypes.byref(st.desc), ctypes.byref(queue.desc), ctypes.byref(plan)), "dp_fifo_plan")
        if plan.done:
            break
        if plan.push_before >= 0:
            push_block(plan.push_before)
            _check(_lib.dp_fifo_commit(ctypes.byref(st.desc), ctypes.byref(plan)), "dp_fifo_commit")
            continue
        if fresh_t is not None and plan.ctx_rows:
            first = (plan.ctx_rows - lat.data_ptr()) // lat.element_size()
            ctx = lat.view(-1)[first:first + plan.ctx_n * lat.shape[2]].view(plan.ctx_n, lat.shape[2])
            context_refresh(ctx, ctx, blocks_from_table(table, [fresh_t], [plan.ctx_n]), cache, stream=stream)
        blk, win, n = queue_blocks(queue, table, tau)
        push = plan.push_after if plan.push_after >= 0 else None
        fused_push = push is not None and frame_pool is None
        o = out[st.step % len(out)] if isinstance(out, (list, tuple)) else out
        window_step(win, win, win, blk, cache, kv_work, o[:n], n_heads, head_dim, pop=bool(plan.pop), queue=queue,
                    push_noise=noise_blocks[push] if fused_push else None, stream=stream, n_win=n,
                    cache_all_slots=cache_all_slots)
        if push is not None and not fused_push:
            push_block(push)
        if on_step is not None:
            on_step(st.step, n, bool(plan.pop), push)
        _check(_lib.dp_fifo_commit(ctypes.byref(st.desc), ctypes.byref(plan)), "dp_fifo_commit")
        run += 1
    return st.step


class FifoState:
    """Progress of a run_fifo run (the library's dp_fifo schedule): steps taken, the next
    block to push (0 = none pushed yet) and the row count of the block that left last."""

    def __init__(self, step: int = 0, nxt: int = 0, exited_rows: int = 0):
        self.desc = DpFifo()
        self.desc.step, self.desc.next_block, self.desc.exited_rows = step, nxt, exited_rows

    def bind(self, n_blocks: int, n_timesteps: int, window_blocks: int) -> None:
        """Attach the schedule's sizes (dp_fifo_init for a fresh run, the saved progress kept)."""
        step, nxt, ex = self.step, self.nxt, self.exited_rows
        _check(_lib.dp_fifo_init(ctypes.byref(self.desc), int(n_blocks), int(n_timesteps), int(window_blocks)),
               "dp_fifo_init")
        self.desc.step, self.desc.next_block, self.desc.exited_rows = step, nxt, ex

    step = property(lambda self: self.desc.step)
    nxt = property(lambda self: self.desc.next_block)
    exited_rows = property(lambda self: self.desc.exited_rows)


_QUEUE_FIELDS = ("slot_rows", "hidden", "n_slots", "head", "count", "n_pushed", "n_popped", "dtype")
_CACHE_FIELDS = ("capacity", "hidden", "n_slots", "n_advances", "dtype")


def checkpoint(queue: Queue, cache: KVCache, state: Optional[FifoState] = None) -> dict:
    """Host copy of a run's state: the queue's and the cache's descriptors and device buffers
    (copied to host memory after the work enqueued on the current stream), and the run's
    progress.  The dict holds plain values and CPU tensors (torch.save-able)."""
    qd, cd = queue.desc, cache.desc
    return {
        "queue": {**{f: getattr(qd, f) for f in _QUEUE_FIELDS},
                  "rows": list(qd.rows), "evals": list(qd.evals)},
        "queue_latent": queue.latent.cpu(),
        "cache": {**{f: getattr(cd, f) for f in _CACHE_FIELDS}, "len": list(cd.len)},
        "cache_k": cache.k.cpu(),
        "cache_v": cache.v.cpu(),
        "state": None if state is None else {"step": state.step, "nxt": state.nxt, "exited_rows": state.exited_rows},
    }


def restore(ckpt: dict, device="cuda"):
    """(queue, cache, state) rebuilt from checkpoint(): new device buffers holding the saved
    bytes, descriptors with the saved fields."""
    q, c = ckpt["queue"], ckpt["cache"]
    lat = ckpt["queue_latent"]
    queue = Queue(q["n_slots"], q["slot_rows"], q["hidden"], dtype=lat.dtype, device=device)
    queue.latent.copy_(lat)
    for f in _QUEUE_FIELDS:
        setattr(queue.desc, f, q[f])
    for i in range(MAX_SLOTS):
        queue.desc.rows[i], queue.desc.evals[i] = q["rows"][i], q["evals"][i]
    k, v = ckpt["cache_k"], ckpt["cache_v"]
    cache = KVCache(c["capacity"], c["hidden"], dtype=k.dtype, n_slots=c["n_slots"], device=device)
    cache.k.copy_(k)
    cache.v.copy_(v)
    for f in _CACHE_FIELDS:
        setattr(cache.desc, f, c[f])
    for i in range(MAX_SLOTS):
        cache.desc.len[i] = c["len"][i]
    st = ckpt["state"]
    return queue, cache, None if st is None else FifoState(**st)
