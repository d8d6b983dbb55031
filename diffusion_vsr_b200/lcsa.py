"""ctypes binding of ``liblcsa.so`` (declarations in ``include/lcsa.h``).

Argument marshalling only: every step of the path runs in the CUDA kernels of
the library.  Tensors are torch CUDA tensors, passed by data pointer on the
current stream.  There is no CPU fallback: loading fails loudly when the
library is missing.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from . import build as _build

LCSA_OK = 0
LCSA_ERR_INVALID_ARG = 1
LCSA_ERR_UNSUPPORTED_DEVICE = 2
LCSA_ERR_CUDA = 3
LCSA_ERR_TIMEOUT = 4
LCSA_ERR_BAD_INDEX = 8
LCSA_FLAG_FORCE_TIMEOUT = 1
LCSA_FLAG_PDL = 2
LCSA_MAX_CANDIDATES = 4096
LCSA_MAX_SEGMENTS = 256

EXPORTED_SYMBOLS = ("lcsa_cache_append", "lcsa_draft_mask", "lcsa_attention", "lcsa_segment_mask",
                    "lcsa_status_string", "lcsa_version")


class lcsa_rope(ctypes.Structure):
    _fields_ = [("base", ctypes.c_float), ("frame0", ctypes.c_int32)]


class lcsa_params(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("q_layers", ctypes.c_int32), ("local_range", ctypes.c_int32),
                ("local_mode", ctypes.c_int32), ("topk", ctypes.c_int32), ("scale", ctypes.c_float),
                ("flags", ctypes.c_int32), ("rope", lcsa_rope)]


class lcsa_kv_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("kmean", ctypes.c_void_p),
                ("capacity", ctypes.c_int32), ("oldest", ctypes.c_int32), ("count", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("window", ctypes.c_int32), ("appended", ctypes.c_int32)]


class LcsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


_LIB: Optional[ctypes.CDLL] = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load liblcsa.so (built in-tree by ``diffusion_vsr_b200.build``)."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    path = path or _build.LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"LCSA CUDA library not built: {path} is missing "
                           "(run `python -m diffusion_vsr_b200.build`)")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    vp = ctypes.c_void_p
    lib.lcsa_cache_append.argtypes = [P(lcsa_kv_cache), vp, vp, ctypes.c_int32, ctypes.c_int32, P(lcsa_rope), vp,
                                      vp]
    lib.lcsa_cache_append.restype = ctypes.c_int
    lib.lcsa_draft_mask.argtypes = [P(lcsa_params), vp, P(lcsa_kv_cache), vp, vp, vp, vp, vp, vp, vp]
    lib.lcsa_draft_mask.restype = ctypes.c_int
    lib.lcsa_attention.argtypes = [P(lcsa_params), vp, P(lcsa_kv_cache), vp, vp, vp, vp, vp, vp]
    lib.lcsa_attention.restype = ctypes.c_int
    lib.lcsa_segment_mask.argtypes = [P(ctypes.c_int32), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp, vp, vp]
    lib.lcsa_segment_mask.restype = ctypes.c_int
    lib.lcsa_status_string.argtypes = [ctypes.c_int]
    lib.lcsa_status_string.restype = ctypes.c_char_p
    lib.lcsa_version.argtypes = []
    lib.lcsa_version.restype = ctypes.c_int
    if path == _build.LIB_PATH:
        _LIB = lib
    return lib


def status_string(code: int) -> str:
    return load_library().lcsa_status_string(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("LCSA tensors must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("LCSA tensors must be contiguous")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(fn: str, rc: int) -> None:
    if rc != LCSA_OK:
        raise LcsaError(fn, rc)


def make_params(heads: int, grid_h: int, grid_w: int, q_layers: int, topk: int, local_range: int = 11,
                local_mode: int = 0, scale: float = 0.0, flags: int = 0, rope_base: float = 0.0,
                rope_frame0: int = 0) -> lcsa_params:
    return lcsa_params(heads, 128, grid_h, grid_w, q_layers, local_range, local_mode, topk, scale, flags,
                       lcsa_rope(rope_base, rope_frame0))


@dataclass
class KVCache:
    """Caller-owned ring buffers (torch CUDA tensors) plus the C descriptor."""
    k: torch.Tensor       # bf16 [capacity, H, nblk, 128, 128]
    v: torch.Tensor
    kmean: torch.Tensor   # fp32 [capacity, H, nblk, 128]
    desc: lcsa_kv_cache

    @classmethod
    def allocate(cls, capacity: int, heads: int, grid_h: int, grid_w: int, device="cuda",
                 window: int = 0) -> "KVCache":
        """``capacity`` slots of which at most ``window`` layers are resident (0: all)."""
        nblk = grid_h * grid_w
        k = torch.empty((capacity, heads, nblk, 128, 128), dtype=torch.bfloat16, device=device)
        v = torch.empty_like(k)
        km = torch.empty((capacity, heads, nblk, 128), dtype=torch.float32, device=device)
        desc = lcsa_kv_cache(k.data_ptr(), v.data_ptr(), km.data_ptr(), capacity, 0, 0, heads, grid_h, grid_w,
                             window)
        return cls(k, v, km, desc)

    @property
    def count(self) -> int:
        return self.desc.count

    @property
    def oldest(self) -> int:
        return self.desc.oldest

    def slot_of_layer(self, layer: int) -> int:
        return (self.desc.oldest + layer) % self.desc.capacity

    def reset(self) -> None:
        self.desc.oldest = 0
        self.desc.count = 0
        self.desc.appended = 0


def lcsa_cache_append(cache: KVCache, k_tok: torch.Tensor, v_tok: torch.Tensor, n_layers: Optional[int] = None,
                      d_status: Optional[torch.Tensor] = None, stream=None, flags: int = 0,
                      rope: Optional[lcsa_rope] = None) -> None:
    if n_layers is None:
        n_layers = k_tok.shape[1] // 2
    rc = load_library().lcsa_cache_append(ctypes.byref(cache.desc), _ptr(k_tok), _ptr(v_tok), n_layers, flags,
                                          ctypes.byref(rope) if rope is not None else None, _ptr(d_status),
                                          _stream(stream))
    _check("lcsa_cache_append", rc)


def lcsa_draft_mask(params: lcsa_params, q_tok: torch.Tensor, cache: KVCache, kept_idx: torch.Tensor,
                    kept_cnt: torch.Tensor, scores: Optional[torch.Tensor] = None,
                    qmean: Optional[torch.Tensor] = None, d_status: Optional[torch.Tensor] = None,
                    stream=None, q_rot: Optional[torch.Tensor] = None) -> None:
    rc = load_library().lcsa_draft_mask(ctypes.byref(params), _ptr(q_tok), ctypes.byref(cache.desc),
                                        _ptr(kept_idx), _ptr(kept_cnt), _ptr(scores), _ptr(qmean), _ptr(q_rot),
                                        _ptr(d_status), _stream(stream))
    _check("lcsa_draft_mask", rc)


def lcsa_attention(params: lcsa_params, q_tok: torch.Tensor, cache: KVCache, kept_idx: torch.Tensor,
                   kept_cnt: torch.Tensor, out_tok: torch.Tensor, lse: Optional[torch.Tensor] = None,
                   d_status: Optional[torch.Tensor] = None, stream=None) -> None:
    rc = load_library().lcsa_attention(ctypes.byref(params), _ptr(q_tok), ctypes.byref(cache.desc),
                                       _ptr(kept_idx), _ptr(kept_cnt), _ptr(out_tok), _ptr(lse),
                                       _ptr(d_status), _stream(stream))
    _check("lcsa_attention", rc)


def lcsa_segment_mask(seg_tiles, heads: int, kept_idx: torch.Tensor, kept_cnt: torch.Tensor,
                      stream=None) -> None:
    """Kept lists of segment-masked dense attention; ``seg_tiles`` is a host sequence."""
    n = len(seg_tiles)
    arr = (ctypes.c_int32 * max(n, 1))(*seg_tiles)
    rc = load_library().lcsa_segment_mask(arr, n, heads, kept_idx.shape[-1], _ptr(kept_idx), _ptr(kept_cnt),
                                          _stream(stream))
    _check("lcsa_segment_mask", rc)


class SegmentAttention:
    """Segment-masked dense attention over a packed sequence of clips.

    The Stage-1 teacher's attention (every token attends to its own segment
    only) as three library calls: the packed k/v appended as one block-layer
    per 128-token tile to a ring of grid 1 x 1, the kept lists of the segment
    table, and the block-sparse attention over them.  q, k, v, out: bf16
    [heads, 128 * tiles, 128] on the GPU, every segment a whole number of tiles.
    """

    def __init__(self, heads: int, seg_tiles, device="cuda"):
        self.seg_tiles = [int(t) for t in seg_tiles]
        self.tiles = sum(self.seg_tiles)
        self.topk = max(self.seg_tiles)
        self.heads = heads
        self.cache = KVCache.allocate(self.tiles, heads, 1, 1, device)
        self.params = make_params(heads, 1, 1, self.tiles, self.topk, local_range=0)
        self.kept_idx = torch.empty((heads, self.tiles, self.topk), dtype=torch.int32, device=device)
        self.kept_cnt = torch.empty((heads, self.tiles), dtype=torch.int32, device=device)
        self.status = torch.zeros((1,), dtype=torch.int32, device=device)
        lcsa_segment_mask(self.seg_tiles, heads, self.kept_idx, self.kept_cnt)

    def run(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
            lse: Optional[torch.Tensor] = None) -> None:
        shape = (self.heads, 128 * self.tiles, 128)
        for t in (q, k, v, out):
            if tuple(t.shape) != shape:
                raise ValueError(f"expected {shape}, got {tuple(t.shape)}")
        self.cache.reset()
        lcsa_cache_append(self.cache, k, v, n_layers=self.tiles, d_status=self.status)
        lcsa_attention(self.params, q, self.cache, self.kept_idx, self.kept_cnt, out, lse, d_status=self.status)


class LcsaLayer:
    """One LCSA attention layer of a streaming DiT: cache + draft + attention.

    Owns the ring and the per-step buffers; ``step`` appends the chunk's k/v,
    builds the draft mask and runs the block-sparse attention, all on the
    current stream.
    """

    def __init__(self, heads: int, grid_h: int, grid_w: int, q_layers: int, kv_len: int, topk: int,
                 local_range: int = 11, local_mode: int = 0, device="cuda", rope_base: float = 0.0):
        self.params = make_params(heads, grid_h, grid_w, q_layers, topk, local_range, local_mode,
                                  rope_base=rope_base)
        # step(): the draft follows the append and the attention the draft, neither of
        # which writes q or the output, so both may launch as programmatic dependents
        self.params_chained = make_params(heads, grid_h, grid_w, q_layers, topk, local_range, local_mode,
                                          flags=LCSA_FLAG_PDL, rope_base=rope_base)
        # with RoPE the draft stores the q it rotates, and the attention reads that
        # copy without rotating again (params without a rotation)
        self.params_attn = make_params(heads, grid_h, grid_w, q_layers, topk, local_range, local_mode,
                                       flags=LCSA_FLAG_PDL)
        self.q_rot: Optional[torch.Tensor] = None
        # kv_len + q_layers resident layers plus q_layers spare slots: a step's append
        # never overwrites a layer the previous step reads (see step(overlap_previous))
        self.cache = KVCache.allocate(kv_len + 2 * q_layers, heads, grid_h, grid_w, device,
                                      window=kv_len + q_layers)
        nq = q_layers * grid_h * grid_w
        self.kept_idx = torch.empty((heads, nq, topk), dtype=torch.int32, device=device)
        self.kept_cnt = torch.empty((heads, nq), dtype=torch.int32, device=device)
        self.status = torch.zeros((1,), dtype=torch.int32, device=device)
        self.rope_base = rope_base
        self.frame = 0  # stream position of the next appended frame (RoPE time axis)

    def _rope(self, frame0: int) -> Optional[lcsa_rope]:
        return lcsa_rope(self.rope_base, frame0) if self.rope_base else None

    def append(self, k_tok: torch.Tensor, v_tok: torch.Tensor) -> None:
        lcsa_cache_append(self.cache, k_tok, v_tok, d_status=self.status, rope=self._rope(self.frame))
        self.frame += k_tok.shape[1]

    def step(self, q_tok: torch.Tensor, k_tok: torch.Tensor, v_tok: torch.Tensor, out_tok: torch.Tensor,
             lse: Optional[torch.Tensor] = None, overlap_previous: bool = False) -> None:
        """Append the chunk's k/v, build the draft mask, run the attention.

        overlap_previous: the kernel before this call in the stream is the previous
        step's attention (or anything else that writes neither k_tok nor v_tok);
        the append is then launched as its programmatic dependent and runs in the
        SMs that attention's last CTAs leave idle.
        """
        frame0 = self.frame
        lcsa_cache_append(self.cache, k_tok, v_tok, d_status=self.status,
                          flags=LCSA_FLAG_PDL if overlap_previous else 0, rope=self._rope(frame0))
        self.frame += k_tok.shape[1]
        self.params.rope.frame0 = frame0
        self.params_chained.rope.frame0 = frame0
        if not self.rope_base:
            lcsa_draft_mask(self.params_chained, q_tok, self.cache, self.kept_idx, self.kept_cnt,
                            d_status=self.status)
            lcsa_attention(self.params_chained, q_tok, self.cache, self.kept_idx, self.kept_cnt, out_tok, lse,
                           d_status=self.status)
            return
        if self.q_rot is None or self.q_rot.shape != q_tok.shape:
            self.q_rot = torch.empty_like(q_tok)
        lcsa_draft_mask(self.params_chained, q_tok, self.cache, self.kept_idx, self.kept_cnt, d_status=self.status,
                        q_rot=self.q_rot)
        lcsa_attention(self.params_attn, self.q_rot, self.cache, self.kept_idx, self.kept_cnt, out_tok, lse,
                       d_status=self.status)


class HostStream:
    """Host-fed streaming over an :class:`LcsaLayer` with copies overlapped.

    Chunk i's q/k/v are copied from pinned host memory on a copy stream while
    chunk i-1 computes, and chunk i-1's output is copied back on a second copy
    stream while chunk i computes: two device slots per buffer, ordered by
    CUDA events (no host synchronisation).  Each ``submit`` enqueues one chunk
    (append + draft + attention through the C ABI) and returns at once; the
    host output buffer of chunk i is complete once ``done(i)`` is.
    """

    def __init__(self, layer: LcsaLayer, q_shape, device="cuda", depth: int = 2):
        self.layer = layer
        self.device = torch.device(device)
        self.depth = depth
        self.compute = torch.cuda.current_stream(self.device)
        self.copy_in = torch.cuda.Stream(self.device)
        self.copy_out = torch.cuda.Stream(self.device)
        mk = lambda: torch.empty(q_shape, dtype=torch.bfloat16, device=self.device)
        self.inputs = [(mk(), mk(), mk()) for _ in range(depth)]
        self.outputs = [mk() for _ in range(depth)]
        ev = lambda: torch.cuda.Event()
        self.in_ready = [ev() for _ in range(depth)]
        self.computed = [ev() for _ in range(depth)]
        self.copied_out = [ev() for _ in range(depth)]
        for e in self.computed + self.copied_out:  # every slot starts free
            e.record(self.compute)
        self._n = 0

    def submit(self, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
               out_host: torch.Tensor) -> int:
        i = self._n
        b = i % self.depth
        q, k, v = self.inputs[b]
        # copy in once the chunk that last used this slot finished computing
        self.copy_in.wait_event(self.computed[b])
        with torch.cuda.stream(self.copy_in):
            q.copy_(q_host, non_blocking=True)
            k.copy_(k_host, non_blocking=True)
            v.copy_(v_host, non_blocking=True)
            self.in_ready[b].record(self.copy_in)
        # compute once the inputs landed and the slot's previous output left
        self.compute.wait_event(self.in_ready[b])
        self.compute.wait_event(self.copied_out[b])
        with torch.cuda.stream(self.compute):
            # the kernel before this step on the compute stream is the previous
            # chunk's attention (or none): the append may overlap it
            self.layer.step(q, k, v, self.outputs[b], overlap_previous=True)
        self.computed[b].record(self.compute)
        self.copy_out.wait_event(self.computed[b])
        with torch.cuda.stream(self.copy_out):
            out_host.copy_(self.outputs[b], non_blocking=True)
            self.copied_out[b].record(self.copy_out)
        self._n += 1
        return i

    def done(self, i: int) -> torch.cuda.Event:
        """Event after which chunk i's output is in its host buffer (valid until chunk i + depth is submitted)."""
        return self.copied_out[i % self.depth]

    def drain_into(self, stream: torch.cuda.Stream) -> None:
        """Make ``stream`` wait for every copy and computation submitted so far."""
        for e in self.copied_out:
            stream.wait_event(e)
