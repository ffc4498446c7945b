"""Thin ctypes binding of ``libpaged.so`` (C ABI in ``include/paged.h``).

Argument marshalling only: tensors are passed as raw device pointers plus
sizes, on torch's current CUDA stream.  Every step of the computation runs in
the library's kernels.  There is no fallback: without the built library, or
with a tensor that is not on a CUDA device, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libpaged.so")

PA_F16, PA_BF16 = 0, 1
PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_WORKSPACE, PA_ERR_OUT_OF_BLOCKS = range(6)

ERRF_SLOT_RANGE = 1 << 0
ERRF_BLOCK_RANGE = 1 << 1
ERRF_CONTEXT = 1 << 2
ERRF_TIMEOUT = 1 << 3

SYMBOLS = ("pa_reshape_and_cache", "pa_decode_workspace_size", "pa_decode", "pa_decode_static",
           "pa_decode_step_host", "pa_decode_step_host_pipelined", "pa_step_inputs_layout", "pa_prefill", "pa_prefill_mma", "pa_copy_blocks", "pa_swap_blocks", "pa_bm_create",
           "pa_bm_destroy", "pa_bm_num_free_blocks", "pa_bm_add_sequence", "pa_bm_fork", "pa_bm_append_slot",
           "pa_bm_free_sequence", "pa_bm_context_len", "pa_bm_block_table", "pa_bm_blocks_needed_to_append",
           "pa_bm_prepare_decode", "pa_bm_swap_sequence", "pa_selftest_wait_timeout", "pa_selftest_exp2", "pa_status_string",
           "pa_version", "pa_last_error")

_lib: Optional[ctypes.CDLL] = None

_c = ctypes
_vp, _i32, _i64, _f32, _sz = _c.c_void_p, _c.c_int, _c.c_int64, _c.c_float, _c.c_size_t


class LibpagedError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status in (PA_ERR_CUDA, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE):
            detail = " [" + load().pa_last_error().decode(errors="replace") + "]"
        super().__init__(f"{where}: {status_string(status)}{detail}")


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (once) and return the shared library."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FileNotFoundError(
            f"{p} is not built; run `python -m paged_kv_cache_368_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(p)
    lib.pa_reshape_and_cache.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i64, _i32, _vp, _vp]
    lib.pa_reshape_and_cache.restype = _i32
    lib.pa_decode_workspace_size.argtypes = [_i32, _i32, _i32, _i32, _i32]
    lib.pa_decode_workspace_size.restype = _sz
    lib.pa_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _f32, _i32, _i32, _i32, _i32, _i64,
                              _i32, _vp, _sz, _i32, _vp, _vp]
    lib.pa_decode.restype = _i32
    lib.pa_decode_static.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _f32, _i32, _i32, _i32, _i32,
                                     _i64, _i32, _i32, _vp, _vp]
    lib.pa_decode_static.restype = _i32
    lib.pa_step_inputs_layout.argtypes = [_i32, _i32, _i32, _i32, _i32, _c.POINTER(_sz)]
    lib.pa_step_inputs_layout.restype = _sz
    lib.pa_decode_step_host.argtypes = [_vp] * 6 + [_i32, _i32, _i32, _f32, _i32, _i32, _i32, _i32, _i64, _i32,
                                                    _vp, _sz, _vp, _vp]
    lib.pa_decode_step_host.restype = _i32
    lib.pa_decode_step_host_pipelined.argtypes = [_vp] * 6 + [_i32, _i32, _i32, _f32, _i32, _i32, _i32, _i32, _i64,
                                                              _i32, _vp, _sz, _vp] + [_vp] * 7
    lib.pa_decode_step_host_pipelined.restype = _i32
    for f in ("pa_prefill", "pa_prefill_mma"):
        getattr(lib, f).argtypes = [_vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _f32, _i32, _i32,
                                    _i32, _i32, _i64, _i32, _vp, _vp]
        getattr(lib, f).restype = _i32
    lib.pa_selftest_wait_timeout.argtypes = [_c.c_uint64, _vp, _vp]
    lib.pa_selftest_wait_timeout.restype = _i32
    lib.pa_selftest_exp2.argtypes = [_vp, _vp, _vp, _i64, _vp]
    lib.pa_selftest_exp2.restype = _i32
    lib.pa_status_string.argtypes = [_i32]
    lib.pa_status_string.restype = _c.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = _i32
    lib.pa_last_error.argtypes = []
    lib.pa_last_error.restype = _c.c_char_p
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().pa_status_string(int(status)).decode()


def dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.float16:
        return PA_F16
    if dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"libpaged supports float16 and bfloat16, not {dtype}")


def _dev_ptr(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libpaged has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      slot_mapping: torch.Tensor, err_flags: Optional[torch.Tensor] = None, stream=None) -> None:
    """Append: ``k_cache[s // bs, :, s % bs, :] = key[n]`` for ``s = slot_mapping[n] >= 0`` (same for V).

    key/value ``[T, KVH, D]``; caches ``[NB, KVH, BS, D]``; slot_mapping int64 ``[T]``."""
    if k_cache.dim() != 4 or key.dim() != 3:
        raise ValueError("k_cache must be [NB, KVH, BS, D] and key [T, KVH, D]")
    nb, kvh, bs, d = k_cache.shape
    if key.shape[1:] != (kvh, d) or value.shape != key.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between key/value and the caches")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (key.shape[0],):
        raise ValueError("slot_mapping must be int64 [T]")
    if not (key.dtype == value.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("key, value and caches must share one dtype")
    st = load().pa_reshape_and_cache(
        _dev_ptr(key, "key"), _dev_ptr(value, "value"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
        _dev_ptr(slot_mapping, "slot_mapping"), key.shape[0], kvh, d, bs, nb, dtype_code(key.dtype),
        _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_reshape_and_cache")


def decode_workspace_size(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int,
                          max_context_len: int) -> int:
    return int(load().pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len))


def alloc_workspace(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int, max_context_len: int,
                    device=None) -> torch.Tensor:
    """A decode workspace, zero-filled as pa_decode requires before its first
    use (every call leaves it zeroed again where that matters)."""
    n = decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len)
    if n == 0:
        raise LibpagedError(PA_ERR_UNSUPPORTED, "pa_decode_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device if device is not None else "cuda")


def decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
           max_context_len: Optional[int] = None, workspace: Optional[torch.Tensor] = None, max_ctas: int = 0,
           err_flags: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``out[s, h] = softmax(scale * q[s, h] . K_s^T) V_s`` over the paged caches.

    q/out ``[S, H, D]``; caches ``[NB, KVH, BS, D]``; block_tables int32 ``[S, MB]``;
    context_lens int32 ``[S]`` (counting the token appended this step).
    ``max_context_len`` bounds context_lens (default ``MB * BS``, no device sync)."""
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [S, H, D] and k_cache [NB, KVH, BS, D]")
    S, H, D = q.shape
    nb, kvh, bs, d2 = k_cache.shape
    if d2 != D or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch between q/out and the caches")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("block_tables must be int32 [S, MB]")
    if context_lens.dtype != torch.int32 or context_lens.shape != (S,):
        raise ValueError("context_lens must be int32 [S]")
    if not (q.dtype == out.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q, out and caches must share one dtype")
    mb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = mb * bs
    if workspace is None:
        workspace = alloc_workspace(S, H, kvh, D, max_context_len, device=q.device)
    st = load().pa_decode(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
        _dev_ptr(block_tables, "block_tables"), mb, _dev_ptr(context_lens, "context_lens"), S,
        int(max_context_len), float(scale), H, kvh, D, bs, nb, dtype_code(q.dtype),
        _dev_ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(), int(max_ctas),
        _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_decode")
    return out


def decode_static(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                  max_context_len: Optional[int] = None, max_ctas: int = 0,
                  err_flags: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``decode`` without a workspace, for callers that cannot allocate device
    memory: the library's own fixed 10 MiB scratch array is used instead.
    Calls that may run concurrently on one GPU race on that array; make the
    first call on a device before any stream capture."""
    S, H, D = q.shape
    nb, kvh, bs, _ = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q/out and the caches")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    mb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = mb * bs
    st = load().pa_decode_static(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
        _dev_ptr(block_tables, "block_tables"), mb, _dev_ptr(context_lens, "context_lens"), S,
        int(max_context_len), float(scale), H, kvh, D, bs, nb, dtype_code(q.dtype), int(max_ctas),
        _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_decode_static")
    return out


def _host_ptr(t: torch.Tensor, name: str) -> int:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


STEP_INPUTS = ("q", "key", "value", "slot_mapping", "block_tables", "context_lens")


def step_inputs_layout(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int, max_blocks_per_seq: int):
    """(offsets, total bytes) of the packed per-step inputs of ``decode_step_host``."""
    off = (_sz * 6)()
    total = load().pa_step_inputs_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq, off)
    if total == 0:
        raise LibpagedError(PA_ERR_INVALID, "pa_step_inputs_layout")
    return dict(zip(STEP_INPUTS, list(off))), int(total)


def pack_step_inputs(buf: torch.Tensor, offsets: dict, **tensors) -> torch.Tensor:
    """Copy host tensors into their slots of a packed uint8 staging buffer."""
    for name, t in tensors.items():
        raw = t.contiguous().view(torch.uint8).reshape(-1)
        buf[offsets[name]: offsets[name] + raw.numel()].copy_(raw)
    return buf


def decode_step_host(h_inputs: torch.Tensor, d_inputs: torch.Tensor, h_out: torch.Tensor, d_out: torch.Tensor,
                     k_cache: torch.Tensor, v_cache: torch.Tensor, num_heads: int, max_blocks_per_seq: int,
                     scale: float, max_context_len: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
                     err_flags: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step from a packed host staging buffer (pinned for
    asynchronous copies): copy in, append the new K/V, decode, copy the
    output to ``h_out``.  Returns ``h_out``; valid once the stream is
    synchronized."""
    S = h_out.shape[0]
    nb, kvh, bs, D = k_cache.shape
    if max_context_len is None:
        max_context_len = max_blocks_per_seq * bs
    if workspace is None:
        workspace = alloc_workspace(S, num_heads, kvh, D, max_context_len, device=k_cache.device)
    st = load().pa_decode_step_host(
        _host_ptr(h_inputs, "h_inputs"), _dev_ptr(d_inputs, "d_inputs"), _host_ptr(h_out, "h_out"),
        _dev_ptr(d_out, "d_out"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), S, max_blocks_per_seq,
        int(max_context_len), float(scale), num_heads, kvh, D, bs, nb, dtype_code(k_cache.dtype),
        _dev_ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_decode_step_host")
    return h_out


class StepPipeline:
    """Host-driven decode steps whose copies overlap the neighbouring steps'
    kernels (pa_decode_step_host_pipelined): the input copy of step i+1 runs
    on ``in_stream`` while step i computes, the output copy of step i on
    ``out_stream`` while step i+1 computes.  Two sets of device staging
    buffer, device output buffer and four events are used in turn."""

    def __init__(self, staging_bytes: int, out_shape, dtype: torch.dtype, device=None, stream=None, in_stream=None,
                 out_stream=None):
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        self.in_stream = in_stream if in_stream is not None else torch.cuda.Stream(dev)
        self.out_stream = out_stream if out_stream is not None else torch.cuda.Stream(dev)
        self.d_inputs = [torch.empty(staging_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.d_out = [torch.empty(tuple(out_shape), dtype=dtype, device=dev) for _ in range(2)]
        # per set: inputs_ready, inputs_free, output_ready, output_free
        self.events = [tuple(torch.cuda.Event() for _ in range(4)) for _ in range(2)]
        for evs in self.events:  # creates the events (torch makes them on first record)
            for ev in evs:
                ev.record(self.stream)
        self.step_index = 0

    def args(self, b: int, h_inputs: torch.Tensor, h_out: torch.Tensor, k_cache: torch.Tensor,
             v_cache: torch.Tensor, num_heads: int, max_blocks_per_seq: int, scale: float, max_context_len: int,
             workspace: torch.Tensor, err_flags: Optional[torch.Tensor] = None) -> tuple:
        """The C-ABI arguments of a step that uses set ``b`` (built once and
        reused by a loop that calls the library directly)."""
        S = h_out.shape[0]
        nb, kvh, bs, D = k_cache.shape
        return (_host_ptr(h_inputs, "h_inputs"), _dev_ptr(self.d_inputs[b], "d_inputs"), _host_ptr(h_out, "h_out"),
                _dev_ptr(self.d_out[b], "d_out"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), S,
                max_blocks_per_seq, int(max_context_len), float(scale), num_heads, kvh, D, bs, nb,
                dtype_code(k_cache.dtype), _dev_ptr(workspace, "workspace"),
                workspace.numel() * workspace.element_size(), _dev_ptr(err_flags, "err_flags"),
                self.stream.cuda_stream, self.in_stream.cuda_stream, self.out_stream.cuda_stream,
                *(ev.cuda_event for ev in self.events[b]))

    def step(self, h_inputs: torch.Tensor, h_out: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
             num_heads: int, max_blocks_per_seq: int, scale: float, max_context_len: Optional[int] = None,
             workspace: Optional[torch.Tensor] = None, err_flags: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Enqueue one step; ``h_out`` holds its output after ``wait()``."""
        b = self.step_index % 2
        self.step_index += 1
        S = h_out.shape[0]
        nb, kvh, bs, D = k_cache.shape
        if max_context_len is None:
            max_context_len = max_blocks_per_seq * bs
        if workspace is None:
            workspace = alloc_workspace(S, num_heads, kvh, D, max_context_len, device=k_cache.device)
        st = load().pa_decode_step_host_pipelined(*self.args(b, h_inputs, h_out, k_cache, v_cache, num_heads,
                                                             max_blocks_per_seq, scale, max_context_len, workspace,
                                                             err_flags))
        if st != PA_OK:
            raise LibpagedError(st, "pa_decode_step_host_pipelined")
        return h_out

    def join(self, stream=None) -> None:
        """Make ``stream`` (default: the compute stream) wait for every copy
        enqueued so far, without blocking the host."""
        s = stream if stream is not None else self.stream
        s.wait_stream(self.in_stream)
        s.wait_stream(self.out_stream)

    def wait(self) -> None:
        """Block the host until the last step's output copy has landed."""
        if self.step_index:
            self.events[(self.step_index - 1) % 2][3].synchronize()


# ------------------------------------------------------------------ block operations


def _setup_block_api(lib):
    if getattr(lib, "_block_api", False):
        return lib
    lib.pa_copy_blocks.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _i64, _i32, _vp, _vp]
    lib.pa_copy_blocks.restype = _i32
    lib.pa_swap_blocks.argtypes = [_vp, _i64, _vp, _i64, _i64, _vp, _i64, _vp, _vp]
    lib.pa_swap_blocks.restype = _i32
    P = _vp
    lib.pa_bm_create.argtypes = [_i64, _i32]
    lib.pa_bm_create.restype = P
    lib.pa_bm_destroy.argtypes = [P]
    lib.pa_bm_destroy.restype = None
    lib.pa_bm_num_free_blocks.argtypes = [P]
    lib.pa_bm_num_free_blocks.restype = _i64
    lib.pa_bm_add_sequence.argtypes = [P, _i64, _i64]
    lib.pa_bm_fork.argtypes = [P, _i64, _i64]
    lib.pa_bm_append_slot.argtypes = [P, _i64, _c.POINTER(_i64), _c.POINTER(_i64), _c.POINTER(_i64)]
    lib.pa_bm_free_sequence.argtypes = [P, _i64]
    lib.pa_bm_context_len.argtypes = [P, _i64]
    lib.pa_bm_context_len.restype = _i64
    lib.pa_bm_block_table.argtypes = [P, _i64, _vp, _i32, _c.POINTER(_i32)]
    lib.pa_bm_blocks_needed_to_append.argtypes = [P, _vp, _i32]
    lib.pa_bm_blocks_needed_to_append.restype = _i64
    lib.pa_bm_prepare_decode.argtypes = [P, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _c.POINTER(_i64)]
    lib.pa_bm_swap_sequence.argtypes = [P, P, _i64, _vp, _i64, _c.POINTER(_i64)]
    for f in ("pa_bm_add_sequence", "pa_bm_fork", "pa_bm_append_slot", "pa_bm_free_sequence", "pa_bm_block_table",
              "pa_bm_prepare_decode", "pa_bm_swap_sequence"):
        getattr(lib, f).restype = _i32
    lib._block_api = True
    return lib


def selftest_wait_timeout(err_flags: torch.Tensor, limit_ns: int = 2_000_000, stream=None) -> None:
    """Run the bounded-wait self-test: ``err_flags`` (int32, 2 words, on the
    device) receives ``ERRF_TIMEOUT`` in each word once its wait has given up."""
    if err_flags.dtype != torch.int32 or err_flags.numel() < 2:
        raise ValueError("err_flags must be an int32 device tensor of at least 2 words")
    st = load().pa_selftest_wait_timeout(int(limit_ns), _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_selftest_wait_timeout")


def selftest_exp2(x: torch.Tensor, stream=None):
    """(polynomial 2^x, exp2f(x)) evaluated on the device for a float32 CUDA tensor."""
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    y_poly, y_ref = torch.empty_like(x), torch.empty_like(x)
    st = load().pa_selftest_exp2(_dev_ptr(x, "x"), _dev_ptr(y_poly, "y_poly"), _dev_ptr(y_ref, "y_ref"), x.numel(),
                                 _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_selftest_exp2")
    return y_poly, y_ref


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_pairs: torch.Tensor,
                err_flags: Optional[torch.Tensor] = None, stream=None) -> None:
    """Copy-on-write copies: block ``block_pairs[i, 1]`` of both caches becomes a
    copy of block ``block_pairs[i, 0]``.  ``block_pairs`` int64 ``[n, 2]`` on the device."""
    lib = _setup_block_api(load())
    if block_pairs.dtype != torch.int64:
        raise ValueError("block_pairs must be int64 [n, 2]")
    nb, kvh, bs, d = k_cache.shape
    st = lib.pa_copy_blocks(_dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
                            _dev_ptr(block_pairs, "block_pairs"), block_pairs.numel() // 2, kvh, d, bs, nb,
                            dtype_code(k_cache.dtype), _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_copy_blocks")


def swap_blocks(src_pool: torch.Tensor, dst_pool: torch.Tensor, block_pairs: torch.Tensor,
                err_flags: Optional[torch.Tensor] = None, stream=None) -> None:
    """``dst_pool[block_pairs[i, 1]] = src_pool[block_pairs[i, 0]]`` for pools of
    equal block size; each pool (and the pairs) on the device or in pinned host memory."""
    lib = _setup_block_api(load())
    if src_pool.shape[1:] != dst_pool.shape[1:] or src_pool.dtype != dst_pool.dtype:
        raise ValueError("pools must have the same block shape and dtype")
    for t, name in ((src_pool, "src_pool"), (dst_pool, "dst_pool"), (block_pairs, "block_pairs")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if not t.is_cuda and not t.is_pinned():
            raise ValueError(f"{name} must be on the device or in pinned host memory")
    block_bytes = src_pool[0].numel() * src_pool.element_size()
    st = lib.pa_swap_blocks(src_pool.data_ptr(), src_pool.shape[0], dst_pool.data_ptr(), dst_pool.shape[0],
                            block_bytes, block_pairs.data_ptr(), block_pairs.numel() // 2,
                            _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_swap_blocks")


class BlockManager:
    """Host block manager (C++ in libpaged): free list (lowest id first),
    per-sequence block tables, shared copy-on-write blocks, swapping."""

    def __init__(self, num_blocks: int, block_size: int):
        self._lib = _setup_block_api(load())
        self._h = self._lib.pa_bm_create(num_blocks, block_size)
        if not self._h:
            raise LibpagedError(PA_ERR_INVALID, "pa_bm_create")
        self.num_blocks, self.block_size = num_blocks, block_size

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h:
            self._lib.pa_bm_destroy(h)

    def _check(self, st, where):
        if st != PA_OK:
            raise LibpagedError(st, where)

    @property
    def num_free(self) -> int:
        return int(self._lib.pa_bm_num_free_blocks(self._h))

    def add(self, seq_id: int, num_tokens: int):
        self._check(self._lib.pa_bm_add_sequence(self._h, seq_id, num_tokens), "pa_bm_add_sequence")

    def fork(self, parent: int, child: int):
        self._check(self._lib.pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def append_slot(self, seq_id: int):
        """-> (slot, cow_src, cow_dst)"""
        slot, src, dst = _i64(), _i64(), _i64()
        self._check(self._lib.pa_bm_append_slot(self._h, seq_id, _c.byref(slot), _c.byref(src), _c.byref(dst)),
                    "pa_bm_append_slot")
        return slot.value, src.value, dst.value

    def free(self, seq_id: int):
        self._check(self._lib.pa_bm_free_sequence(self._h, seq_id), "pa_bm_free_sequence")

    def context_len(self, seq_id: int) -> int:
        return int(self._lib.pa_bm_context_len(self._h, seq_id))

    def block_table(self, seq_id: int, max_blocks: int = 1 << 16):
        import numpy as np

        buf = np.empty(max_blocks, dtype=np.int32)
        n = _i32()
        self._check(self._lib.pa_bm_block_table(self._h, seq_id, buf.ctypes.data, max_blocks, _c.byref(n)),
                    "pa_bm_block_table")
        return buf[: n.value].tolist()

    def blocks_needed_to_append(self, seq_ids) -> int:
        import numpy as np

        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        return int(self._lib.pa_bm_blocks_needed_to_append(self._h, ids.ctypes.data, len(ids)))

    def prepare_decode(self, seq_ids, max_blocks_per_seq: int):
        """Append one token to each sequence; -> (block_tables, context_lens, slot_mapping, cow_pairs) numpy."""
        import numpy as np

        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        tables = np.empty((n, max_blocks_per_seq), dtype=np.int32)
        ctx = np.empty(n, dtype=np.int32)
        slots = np.empty(n, dtype=np.int64)
        cow = np.empty((max(n, 1), 2), dtype=np.int64)
        ncow = _i64()
        self._check(self._lib.pa_bm_prepare_decode(self._h, ids.ctypes.data, n, max_blocks_per_seq, tables.ctypes.data,
                                                   ctx.ctypes.data, slots.ctypes.data, cow.ctypes.data,
                                                   _c.byref(ncow)), "pa_bm_prepare_decode")
        return tables, ctx, slots, cow[: ncow.value].copy()

    def swap_to(self, other: "BlockManager", seq_id: int):
        """Move a sequence into `other`'s pool; -> (n, 2) int64 pairs (block here, block there)."""
        import numpy as np

        cap = self.num_blocks
        pairs = np.empty((cap, 2), dtype=np.int64)
        n = _i64()
        self._check(self._lib.pa_bm_swap_sequence(self._h, other._h, seq_id, pairs.ctypes.data, cap, _c.byref(n)),
                    "pa_bm_swap_sequence")
        return pairs[: n.value].copy()


def prefill(out: torch.Tensor, q: torch.Tensor, cu_q_lens: torch.Tensor, k_cache: torch.Tensor,
            v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
            max_q_len: int, max_context_len: Optional[int] = None, err_flags: Optional[torch.Tensor] = None,
            stream=None, legacy_mma: bool = False) -> torch.Tensor:
    """Causal multi-token paged attention (tcgen05 kernel; ``legacy_mma`` runs
    the mma.sync kernel instead).  ``q``/``out`` ``[total_q, H, D]``;
    sequence s owns rows ``cu_q_lens[s]..cu_q_lens[s+1]-1``, which are the last
    tokens of its ``context_lens[s]`` cached positions."""
    T, H, D = q.shape
    nb, kvh, bs, _ = k_cache.shape
    S = context_lens.shape[0]
    if cu_q_lens.dtype != torch.int32 or cu_q_lens.shape != (S + 1,):
        raise ValueError("cu_q_lens must be int32 [S + 1]")
    if out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    mb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = mb * bs
    fn = load().pa_prefill_mma if legacy_mma else load().pa_prefill
    st = fn(
        _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(cu_q_lens, "cu_q_lens"), T, int(max_q_len),
        _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"), mb,
        _dev_ptr(context_lens, "context_lens"), S, int(max_context_len), float(scale), H, kvh, D, bs, nb,
        dtype_code(q.dtype), _dev_ptr(err_flags, "err_flags"), _stream(stream))
    if st != PA_OK:
        raise LibpagedError(st, "pa_prefill")
    return out
