"""Thin ctypes binding of libtp.so (include/tp.h).

Argument marshalling only: torch tensors become device pointers and host
pointer arrays, the current CUDA stream is passed through, and a non-OK status
raises TPError with the library's message. Every step of the computation runs
in the library's kernels; there is no fallback. Importing this module fails
loudly when libtp.so has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtp.so")

TP_F32, TP_BF16 = 0, 1
ACTS = {"none": 0, "gelu": 1, "swiglu": 2}
WHICH = {"mlp": 0, "qkv": 1, "outproj": 2, "vocab": 3}
NORMS = {"layer": 0, "rms": 1}
STATUS = ["TP_OK", "TP_ERR_ARG", "TP_ERR_DIVISIBILITY", "TP_ERR_ALIGN", "TP_ERR_DTYPE",
          "TP_ERR_UNSUPPORTED", "TP_ERR_CUDA", "TP_ERR_TIMEOUT", "TP_ERR_NO_DEVICE"]
MAX_SHARDS = 16


class TPError(RuntimeError):
    def __init__(self, status: int, func: str, msg: str):
        self.status = status
        self.status_name = STATUS[status] if 0 <= status < len(STATUS) else f"status {status}"
        super().__init__(f"{func}: {self.status_name}: {msg}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m megatron_tensor_transformer_gemm_b200.build`")
    return ctypes.CDLL(LIB_PATH)


lib = _load()

_vp = ctypes.c_void_p
_vpp = ctypes.POINTER(ctypes.c_void_p)
_i64 = ctypes.c_int64
_int = ctypes.c_int
_fp = ctypes.c_void_p  # float* (device)
_plan_p = ctypes.c_void_p
_u32 = ctypes.c_uint32

PEER_HANDLE_BYTES = 64
PEER_FLAG_BYTES = 256


class PeerGroupC(ctypes.Structure):
    """tp_peer_group: this rank's view of every rank's flag words and
    receive buffer (device pointers, local or mapped from a peer)."""
    _fields_ = [("world", ctypes.c_int), ("rank", ctypes.c_int), ("recv_elems", ctypes.c_int64),
                ("flags", ctypes.c_void_p * MAX_SHARDS), ("recv", ctypes.c_void_p * MAX_SHARDS)]


_peer_p = ctypes.POINTER(PeerGroupC)

_SIGS = {
    "tp_plan_create": (_int, [_int, _int, _int, _int, _int, _int, _int, ctypes.POINTER(_plan_p)]),
    "tp_plan_destroy": (None, [_plan_p]),
    "tp_plan_describe": (_int, [_plan_p, ctypes.c_char_p, ctypes.c_size_t]),
    "tp_status_string": (ctypes.c_char_p, [_int]),
    "tp_last_error": (ctypes.c_char_p, []),
    "tp_get_device_status": (_int, [_plan_p, _vp]),
    "tp_launch_count": (ctypes.c_uint64, [_int]),
    "tp_selftest_wait_timeout": (_int, [_i64, _vp, _vp]),
    "tp_shard_column": (_int, [_plan_p, _int, _vp, _vpp, _vp]),
    "tp_unshard_column": (_int, [_plan_p, _int, _vpp, _vp, _vp]),
    "tp_shard_row": (_int, [_plan_p, _int, _vp, _vpp, _vp]),
    "tp_unshard_row": (_int, [_plan_p, _int, _vpp, _vp, _vp]),
    "tp_shard_column_bias": (_int, [_plan_p, _int, _vp, _vpp, _vp]),
    "tp_column_fwd": (_int, [_plan_p, _int, _i64, _vp, _vpp, _vpp, _vpp, _vpp, _vp]),
    "tp_row_fwd_partial": (_int, [_plan_p, _int, _i64, _vpp, _vpp, _vpp, _vp]),
    "tp_reduce_partials": (_int, [_plan_p, _i64, _int, _vpp, _vp, _vp, _vp, _vp]),
    "tp_reduce_scatter_seq": (_int, [_plan_p, _i64, _int, _vpp, _vp, _vpp, _vpp, _vp]),
    "tp_all_gather_seq": (_int, [_plan_p, _i64, _int, _vpp, _vp, _vp]),
    "tp_layernorm_fwd": (_int, [_plan_p, _i64, _vp, _vp, _vp, _vp, _fp, _fp, _vp]),
    "tp_layernorm_all_gather_seq": (_int, [_plan_p, _i64, _int, _vpp, _vp, _vp, _vp, _fp, _fp, _vp]),
    "tp_attention_fwd": (_int, [_plan_p, _int, _int, _vpp, _vpp, _vpp, _vp]),
    "tp_row_bwd": (_int, [_plan_p, _int, _i64, _vp, _vpp, _vpp, _vpp, _vpp, _vpp, _fp, _vp]),
    "tp_column_bwd": (_int, [_plan_p, _int, _i64, _vp, _vpp, _vpp, _vpp, _vpp, _vpp, _vp]),
    "tp_reduce_scatter_seq_bwd": (_int, [_plan_p, _i64, _int, _vpp, _vp, _vp]),
    "tp_all_gather_seq_bwd": (_int, [_plan_p, _i64, _int, _vpp, _vpp, _vp]),
    "tp_layernorm_bwd": (_int, [_plan_p, _i64, _vp, _vp, _vp, _fp, _fp, _vp, _vp, _fp, _fp, _int, _vp]),
    "tp_attention_bwd": (_int, [_plan_p, _int, _int, _vpp, _vpp, _vpp, _vpp, _vpp, _vp]),
    "tp_column_sum": (_int, [_plan_p, _i64, _i64, _vp, _fp, _int, _vp]),
    "tp_column_sum_static": (_int, [_i64, _i64, _int, _vp, _fp, _int, _vp]),
    "tp_plan_set_vocab": (_int, [_plan_p, _int, ctypes.POINTER(_int)]),
    "tp_embedding_fwd": (_int, [_plan_p, _i64, _vp, _vpp, _vp, _vp]),
    "tp_embedding_bwd": (_int, [_plan_p, _i64, _vp, _vp, _vpp, _vp]),
    "tp_vocab_cross_entropy": (_int, [_plan_p, _i64, _vpp, _vp, ctypes.c_float, _fp, _fp, _vpp, _vp]),
    "tp_norm_sharded_fwd": (_int, [_plan_p, _int, _i64, _vpp, _vpp, _vpp, _vpp, _fp, _fp, _vp]),
    "tp_norm_sharded_bwd": (_int, [_plan_p, _int, _i64, _vpp, _vpp, _vpp, _fp, _fp, _vpp, _vpp, _vpp, _vp]),
    "tp_row_fwd_reduce": (_int, [_plan_p, _int, _i64, _vpp, _vpp, _vp, _vp, _vp, _vp]),
    "tp_row_fwd_reduce_scatter_seq": (_int, [_plan_p, _int, _i64, _vpp, _vpp, _vp, _vpp, _vpp, _vp]),
    "tp_column_bwd_reduce": (_int, [_plan_p, _int, _i64, _vp, _vpp, _vpp, _vpp, _vpp, _vp, _vp]),
    "tp_column_bwd_reduce_scatter_seq": (_int, [_plan_p, _int, _i64, _vp, _vpp, _vpp, _vpp, _vpp, _vpp, _vp]),
    "tp_set_backward_defer": (_int, [_plan_p, _int]),
    "tp_set_wgrad_grouping": (_int, [_plan_p, _int]),
    "tp_flush_wgrad": (_int, [_plan_p]),
    "tp_backward_join": (_int, [_vp]),
    "tp_peer_alloc": (_int, [ctypes.c_size_t, _vpp, _vp]),
    "tp_peer_free": (_int, [_vp]),
    "tp_peer_open": (_int, [_vp, _vpp]),
    "tp_peer_close": (_int, [_vp]),
    "tp_peer_set_wait_limit": (_int, [_i64]),
    "tp_row_fwd_push_peer": (_int, [_plan_p, _int, _i64, _vpp, _vpp, _peer_p, _u32, _vp]),
    "tp_column_bwd_push_peer": (_int, [_plan_p, _int, _i64, _vp, _vpp, _vpp, _vpp, _vpp, _peer_p, _u32, _vp]),
    "tp_peer_reduce": (_int, [_peer_p, _i64, _int, _vp, _vp, _int, _vpp, _u32, _vp]),
    "tp_peer_wait": (_int, [_peer_p, _u32, _vp]),
    "tp_all_gather_push_peer": (_int, [_peer_p, _i64, _int, _vp, _vpp, _u32, _vp]),
    "tp_layernorm_all_gather_push_peer": (_int, [_plan_p, _peer_p, _i64, _vp, _vp, _vp, _vpp, _fp, _fp, _u32, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def last_error() -> str:
    return (lib.tp_last_error() or b"").decode(errors="replace")


def check(status: int, func: str) -> None:
    if status != 0:
        raise TPError(status, func, last_error())


def launch_count(reset: bool = False) -> int:
    return int(lib.tp_launch_count(1 if reset else 0))


def backward_join(stream=None) -> None:
    """tp_backward_join: the stream waits for the deferred weight gradients
    and bias sums of every plan (see Plan.set_backward_defer)."""
    check(lib.tp_backward_join(_stream(stream)), "tp_backward_join")


def peer_alloc(nbytes: int) -> tuple[int, bytes]:
    """tp_peer_alloc: zeroed device memory other processes can map; returns
    (device pointer, IPC handle bytes)."""
    ptr = ctypes.c_void_p()
    h = ctypes.create_string_buffer(PEER_HANDLE_BYTES)
    check(lib.tp_peer_alloc(nbytes, ctypes.byref(ptr), h), "tp_peer_alloc")
    return ptr.value, h.raw


def peer_free(ptr: int) -> None:
    check(lib.tp_peer_free(ptr), "tp_peer_free")


def peer_open(handle: bytes) -> int:
    """tp_peer_open: map another process's peer memory; returns its pointer here."""
    if len(handle) != PEER_HANDLE_BYTES:
        raise ValueError(f"a peer handle has {PEER_HANDLE_BYTES} bytes, got {len(handle)}")
    ptr = ctypes.c_void_p()
    check(lib.tp_peer_open(ctypes.create_string_buffer(handle, PEER_HANDLE_BYTES), ctypes.byref(ptr)),
          "tp_peer_open")
    return ptr.value


def peer_close(ptr: int) -> None:
    check(lib.tp_peer_close(ptr), "tp_peer_close")


def peer_set_wait_limit(ns: int) -> None:
    check(lib.tp_peer_set_wait_limit(int(ns)), "tp_peer_set_wait_limit")


def peer_group(world: int, rank: int, recv_elems: int, flags: Sequence[int], recv: Sequence[int]) -> PeerGroupC:
    """A tp_peer_group from per-rank device pointers."""
    g = PeerGroupC()
    g.world, g.rank, g.recv_elems = world, rank, recv_elems
    for d in range(world):
        g.flags[d] = flags[d]
        g.recv[d] = recv[d]
    return g


def peer_reduce(g: PeerGroupC, T: int, hidden: int, bias, residual, out: Sequence, epoch: int,
                stream=None) -> None:
    check(lib.tp_peer_reduce(ctypes.byref(g), T, hidden, _ptr(bias), _ptr(residual), len(out), _arr(out),
                             epoch, _stream(stream)), "tp_peer_reduce")


def peer_wait(g: PeerGroupC, epoch: int, stream=None) -> None:
    check(lib.tp_peer_wait(ctypes.byref(g), epoch, _stream(stream)), "tp_peer_wait")


def all_gather_push_peer(g: PeerGroupC, rows: int, cols: int, x, out: Sequence, epoch: int, stream=None) -> None:
    check(lib.tp_all_gather_push_peer(ctypes.byref(g), rows, cols, _ptr(x), _arr(out), epoch, _stream(stream)),
          "tp_all_gather_push_peer")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libtp must be contiguous")
    return t.data_ptr()


def _arr(ts: Sequence | None):
    if ts is None:
        return None
    vals = [_ptr(t) for t in ts]
    return (ctypes.c_void_p * len(vals))(*vals)


def _stream(stream=None) -> int | None:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    if torch.cuda.is_available():
        return torch.cuda.current_stream().cuda_stream
    return None


DTYPES = {"bf16": TP_BF16, "f32": TP_F32}


class Plan:
    """A tp_plan: block dimensions, shard count p, dtype, activation and the
    dtype of the full-shape partial sums (default: the plan dtype)."""

    def __init__(self, hidden: int, ffn: int, heads: int, p: int, dtype: str = "bf16",
                 act: str = "gelu", partial_dtype: str | None = None):
        self.hidden, self.ffn, self.heads, self.p = hidden, ffn, heads, p
        self.dtype_name = dtype
        self.torch_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.partial_dtype_name = partial_dtype or dtype
        self.partial_torch_dtype = torch.bfloat16 if self.partial_dtype_name == "bf16" else torch.float32
        self.act = act
        h = ctypes.c_void_p()
        check(lib.tp_plan_create(hidden, ffn, heads, p, DTYPES[dtype], ACTS[act],
                                 DTYPES[self.partial_dtype_name], ctypes.byref(h)), "tp_plan_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            lib.tp_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def set_vocab(self, vocab: int) -> int:
        """Pad the vocab so the p shards split it; returns the padded size."""
        vp = ctypes.c_int(0)
        check(lib.tp_plan_set_vocab(self._h, vocab, ctypes.byref(vp)), "tp_plan_set_vocab")
        self.vocab, self.vocab_padded = vocab, vp.value
        return vp.value

    def embedding_fwd(self, T, ids, E, Y, stream=None):
        check(lib.tp_embedding_fwd(self._h, T, _ptr(ids), _arr(E), _ptr(Y), _stream(stream)),
              "tp_embedding_fwd")

    def embedding_bwd(self, T, ids, dY, dE, stream=None):
        check(lib.tp_embedding_bwd(self._h, T, _ptr(ids), _ptr(dY), _arr(dE), _stream(stream)),
              "tp_embedding_bwd")

    def vocab_cross_entropy(self, T, logits, labels, grad_scale, loss, lse=None, dlogits=None,
                            stream=None):
        check(lib.tp_vocab_cross_entropy(self._h, T, _arr(logits), _ptr(labels), float(grad_scale),
                                         _ptr(loss), _ptr(lse), _arr(dlogits), _stream(stream)),
              "tp_vocab_cross_entropy")

    def describe(self) -> str:
        buf = ctypes.create_string_buffer(4096)
        check(lib.tp_plan_describe(self._h, buf, len(buf)), "tp_plan_describe")
        return buf.value.decode()

    # ----------------------------------------------------------- sharding
    def shard_column(self, which, W_full, W_shards, stream=None):
        check(lib.tp_shard_column(self._h, WHICH[which], _ptr(W_full), _arr(W_shards), _stream(stream)),
              "tp_shard_column")

    def unshard_column(self, which, W_shards, W_full, stream=None):
        check(lib.tp_unshard_column(self._h, WHICH[which], _arr(W_shards), _ptr(W_full), _stream(stream)),
              "tp_unshard_column")

    def shard_row(self, which, W_full, W_shards, stream=None):
        check(lib.tp_shard_row(self._h, WHICH[which], _ptr(W_full), _arr(W_shards), _stream(stream)),
              "tp_shard_row")

    def unshard_row(self, which, W_shards, W_full, stream=None):
        check(lib.tp_unshard_row(self._h, WHICH[which], _arr(W_shards), _ptr(W_full), _stream(stream)),
              "tp_unshard_row")

    def shard_column_bias(self, which, b_full, b_shards, stream=None):
        check(lib.tp_shard_column_bias(self._h, WHICH[which], _ptr(b_full), _arr(b_shards),
                                       _stream(stream)), "tp_shard_column_bias")

    # ------------------------------------------------------------ forward
    def column_fwd(self, which, T, X, W, bias, Z, H, stream=None):
        check(lib.tp_column_fwd(self._h, WHICH[which], T, _ptr(X), _arr(W), _arr(bias), _arr(Z),
                                _arr(H), _stream(stream)), "tp_column_fwd")

    def row_fwd_partial(self, which, T, H, W, P, stream=None):
        check(lib.tp_row_fwd_partial(self._h, WHICH[which], T, _arr(H), _arr(W), _arr(P),
                                     _stream(stream)), "tp_row_fwd_partial")

    def row_fwd_reduce(self, which, T, H, W, bias, residual, Y, stream=None):
        check(lib.tp_row_fwd_reduce(self._h, WHICH[which], T, _arr(H), _arr(W), _ptr(bias),
                                    _ptr(residual), _ptr(Y), _stream(stream)), "tp_row_fwd_reduce")

    def row_fwd_reduce_scatter_seq(self, which, T, H, W, bias, residual_seq, Y_seq, stream=None):
        check(lib.tp_row_fwd_reduce_scatter_seq(self._h, WHICH[which], T, _arr(H), _arr(W), _ptr(bias),
                                                _arr(residual_seq), _arr(Y_seq), _stream(stream)),
              "tp_row_fwd_reduce_scatter_seq")

    def reduce_partials(self, T, P, bias, residual, Y, stream=None):
        check(lib.tp_reduce_partials(self._h, T, len(P), _arr(P), _ptr(bias), _ptr(residual),
                                     _ptr(Y), _stream(stream)), "tp_reduce_partials")

    def reduce_scatter_seq(self, T, P, bias, residual_seq, Y_seq, stream=None):
        check(lib.tp_reduce_scatter_seq(self._h, T, len(P), _arr(P), _ptr(bias), _arr(residual_seq),
                                        _arr(Y_seq), _stream(stream)), "tp_reduce_scatter_seq")

    def all_gather_seq(self, T, X_seq, X_full, stream=None):
        check(lib.tp_all_gather_seq(self._h, T, len(X_seq), _arr(X_seq), _ptr(X_full),
                                    _stream(stream)), "tp_all_gather_seq")

    def layernorm_fwd(self, rows, x, gamma, beta, y, mean=None, rstd=None, stream=None):
        check(lib.tp_layernorm_fwd(self._h, rows, _ptr(x), _ptr(gamma), _ptr(beta), _ptr(y),
                                   _ptr(mean), _ptr(rstd), _stream(stream)), "tp_layernorm_fwd")

    def layernorm_all_gather_seq(self, T, X_seq, gamma, beta, Y_full, mean=None, rstd=None,
                                 stream=None):
        check(lib.tp_layernorm_all_gather_seq(self._h, T, len(X_seq), _arr(X_seq), _ptr(gamma),
                                              _ptr(beta), _ptr(Y_full), _ptr(mean), _ptr(rstd),
                                              _stream(stream)), "tp_layernorm_all_gather_seq")

    def norm_sharded_fwd(self, kind, rows, X, gamma, beta, Y, mean=None, rstd=None, stream=None):
        """kind: "layer" or "rms"; X, gamma, beta, Y: per-shard tensors (hidden split)."""
        check(lib.tp_norm_sharded_fwd(self._h, NORMS[kind], rows, _arr(X), _arr(gamma), _arr(beta),
                                      _arr(Y), _ptr(mean), _ptr(rstd), _stream(stream)),
              "tp_norm_sharded_fwd")

    def norm_sharded_bwd(self, kind, rows, X, gamma, dY, mean, rstd, dX, dgamma, dbeta=None,
                         stream=None):
        check(lib.tp_norm_sharded_bwd(self._h, NORMS[kind], rows, _arr(X), _arr(gamma), _arr(dY),
                                      _ptr(mean), _ptr(rstd), _arr(dX), _arr(dgamma), _arr(dbeta),
                                      _stream(stream)), "tp_norm_sharded_bwd")

    def attention_fwd(self, batch, seq, QKV, O, LSE=None, stream=None):
        check(lib.tp_attention_fwd(self._h, batch, seq, _arr(QKV), _arr(O), _arr(LSE),
                                   _stream(stream)), "tp_attention_fwd")

    # ----------------------------------------------------------- backward
    def row_bwd(self, which, T, dY, H, W, Z, dZ, dW=None, dbias=None, stream=None):
        check(lib.tp_row_bwd(self._h, WHICH[which], T, _ptr(dY), _arr(H), _arr(W), _arr(Z),
                             _arr(dZ), _arr(dW), _ptr(dbias), _stream(stream)), "tp_row_bwd")

    def column_bwd(self, which, T, X, dZ, W, dW=None, dbias=None, dX_partials=None, stream=None):
        check(lib.tp_column_bwd(self._h, WHICH[which], T, _ptr(X), _arr(dZ), _arr(W), _arr(dW),
                                _arr(dbias), _arr(dX_partials), _stream(stream)), "tp_column_bwd")

    def column_bwd_reduce(self, which, T, X, dZ, W, dW=None, dbias=None, dX=None, stream=None):
        check(lib.tp_column_bwd_reduce(self._h, WHICH[which], T, _ptr(X), _arr(dZ), _arr(W), _arr(dW),
                                       _arr(dbias), _ptr(dX), _stream(stream)), "tp_column_bwd_reduce")

    def layernorm_all_gather_push_peer(self, g: PeerGroupC, rows, x, gamma, beta, out, mean=None, rstd=None,
                                       epoch: int = 0, stream=None):
        check(lib.tp_layernorm_all_gather_push_peer(self._h, ctypes.byref(g), rows, _ptr(x), _ptr(gamma), _ptr(beta),
                                                    _arr(out), _ptr(mean), _ptr(rstd), epoch, _stream(stream)),
              "tp_layernorm_all_gather_push_peer")

    def row_fwd_push_peer(self, which, T, H, W, g: PeerGroupC, epoch: int, stream=None):
        check(lib.tp_row_fwd_push_peer(self._h, WHICH[which], T, _arr(H), _arr(W), ctypes.byref(g), epoch,
                                       _stream(stream)), "tp_row_fwd_push_peer")

    def column_bwd_push_peer(self, which, T, X, dZ, W, dW, dbias, g: PeerGroupC, epoch: int, stream=None):
        check(lib.tp_column_bwd_push_peer(self._h, WHICH[which], T, _ptr(X), _arr(dZ), _arr(W), _arr(dW),
                                          _arr(dbias), ctypes.byref(g), epoch, _stream(stream)),
              "tp_column_bwd_push_peer")

    def column_bwd_reduce_scatter_seq(self, which, T, X, dZ, W, dW=None, dbias=None, dX_seq=None,
                                      stream=None):
        check(lib.tp_column_bwd_reduce_scatter_seq(self._h, WHICH[which], T, _ptr(X), _arr(dZ), _arr(W),
                                                   _arr(dW), _arr(dbias), _arr(dX_seq), _stream(stream)),
              "tp_column_bwd_reduce_scatter_seq")

    def reduce_scatter_seq_bwd(self, T, dY_seq, dY_full, stream=None):
        check(lib.tp_reduce_scatter_seq_bwd(self._h, T, len(dY_seq), _arr(dY_seq), _ptr(dY_full),
                                            _stream(stream)), "tp_reduce_scatter_seq_bwd")

    def all_gather_seq_bwd(self, T, dX_partials, dX_seq, stream=None):
        check(lib.tp_all_gather_seq_bwd(self._h, T, len(dX_partials), _arr(dX_partials),
                                        _arr(dX_seq), _stream(stream)), "tp_all_gather_seq_bwd")

    def layernorm_bwd(self, rows, x, gamma, dy, mean, rstd, dx, dgamma, dbeta, accumulate=False,
                      stream=None, dres=None):
        """dres (optional): a gradient added to dx (the residual branch)."""
        check(lib.tp_layernorm_bwd(self._h, rows, _ptr(x), _ptr(gamma), _ptr(dy), _ptr(mean),
                                   _ptr(rstd), _ptr(dres), _ptr(dx), _ptr(dgamma), _ptr(dbeta),
                                   1 if accumulate else 0, _stream(stream)), "tp_layernorm_bwd")

    def attention_bwd(self, batch, seq, QKV, O, dO, LSE, dQKV, stream=None):
        check(lib.tp_attention_bwd(self._h, batch, seq, _arr(QKV), _arr(O), _arr(dO), _arr(LSE),
                                   _arr(dQKV), _stream(stream)), "tp_attention_bwd")

    def set_wgrad_grouping(self, on: bool = True):
        """tp_set_wgrad_grouping: the row backward's weight gradients wait for
        the next column backward and run in one grouped launch with its own."""
        check(lib.tp_set_wgrad_grouping(self._h, 1 if on else 0), "tp_set_wgrad_grouping")

    def flush_wgrad(self):
        check(lib.tp_flush_wgrad(self._h), "tp_flush_wgrad")

    def set_backward_defer(self, on: bool = True):
        """tp_set_backward_defer: this plan's backward calls leave their weight
        gradients and bias sums on the side stream until backward_join()."""
        check(lib.tp_set_backward_defer(self._h, 1 if on else 0), "tp_set_backward_defer")

    def column_sum(self, rows, cols, x, out, accumulate=False, stream=None):
        check(lib.tp_column_sum(self._h, rows, cols, _ptr(x), _ptr(out), 1 if accumulate else 0,
                                _stream(stream)), "tp_column_sum")


def column_sum_static(rows, cols, x, out, accumulate=False, stream=None):
    """tp_column_sum_static: column sums with the library's fixed device scratch
    (no allocation); see include/tp.h for its limits. x must be a dense
    [rows, cols] tensor (row stride == cols)."""
    dt = TP_BF16 if x.dtype == torch.bfloat16 else TP_F32
    check(lib.tp_column_sum_static(rows, cols, dt, _ptr(x), _ptr(out), 1 if accumulate else 0,
                                   _stream(stream)), "tp_column_sum_static")


def device_status(stream=None, plan: "Plan | None" = None) -> str:
    """Read and clear the device status word: "TP_OK", "TP_ERR_TIMEOUT" (a
    kernel's bounded wait gave up) or "TP_ERR_ARG" (a kernel met an
    out-of-range id or label). A failure to read it raises TPError."""
    st = lib.tp_get_device_status(plan.handle if plan is not None else None, _stream(stream))
    if st in (0, 1, 7):
        return STATUS[st]
    check(st, "tp_get_device_status")
    return STATUS[st]


def selftest_wait_timeout(limit_ns: int, gave_up=None, stream=None) -> None:
    """Launch the library's self-test kernel whose bounded wait runs out after
    limit_ns (<= 1 s): it sets TP_ERR_TIMEOUT in the device status word."""
    check(lib.tp_selftest_wait_timeout(int(limit_ns), _ptr(gave_up), _stream(stream)),
          "tp_selftest_wait_timeout")
