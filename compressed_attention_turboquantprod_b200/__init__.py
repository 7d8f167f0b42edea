"""TurboQuant-prod / QJL compressed KV cache and decode attention on B200 (sm_100a).

The compute lives in ``libtq.so`` (hand-written CUDA kernels behind the C ABI
of ``include/tq.h``); ``native`` is its ctypes binding and this module adds
small owners of the device buffers (allocated with PyTorch) around it.
``native`` is loaded on first use (so that ``build`` can run before the library
exists); using any class here without a built ``libtq.so`` raises ImportError.
"""
from __future__ import annotations

import importlib
import math
from typing import Optional

import torch

__all__ = ["native", "TQError", "Codebook", "Projections", "CompressedKVCache", "LayerGroups",
           "key_variance", "stack_partials", "gather_partials", "merge_partials"]


def __getattr__(name):
    if name == "TQError":
        return importlib.import_module(".native", __name__).TQError
    raise AttributeError(name)


class _Native:
    def __getattr__(self, name):
        return getattr(importlib.import_module(".native", __package__), name)


native = _Native()


class Codebook:
    """Lloyd-Max centroids/boundaries for head dim d and b1 bits, built on the GPU."""

    def __init__(self, d: int, bits: int, device="cuda"):
        self.d, self.bits = d, bits
        L = 1 << bits
        self.centroids = torch.empty(L, dtype=torch.float32, device=device)
        self.boundaries = torch.empty(max(L - 1, 1), dtype=torch.float32, device=device)
        native.tq_codebook_build(d, bits, self.centroids, self.boundaries)


class Projections:
    """Per-layer Pi (d x d), S (m x d) and T = S Pi^T, generated on the GPU.
    structured: the Hadamard rotation Pi = H diag(s) / sqrt(d) instead of the QR one."""

    def __init__(self, d: int, m: int, layer: int, rotation: bool = True, device="cuda",
                 base_seed: int = 42, stride: int = 7, structured: bool = False):
        self.d, self.m, self.layer = d, m, layer
        f32 = dict(dtype=torch.float32, device=device)
        self.Pi = torch.empty(d, d, **f32) if rotation else None
        self.S = torch.empty(m, d, **f32)
        self.T = torch.empty(m, d, **f32)
        if rotation and structured:
            native.tq_make_projections_hadamard(d, m, layer, self.Pi, self.S, self.T, base_seed, stride)
            return
        ws = None
        if rotation:
            ws = torch.empty(native.tq_projections_workspace_bytes(d), dtype=torch.uint8, device=device)
        native.tq_make_projections(d, m, layer, self.Pi, self.S, self.T, ws, base_seed, stride)


class LayerGroups:
    """A-QJL per-layer-group sketch dims from the config strings ("8,16,24", "512,384,256,192")."""

    def __init__(self, boundaries: str, sketch_dims: str):
        self._g = native.tq_layer_groups_parse(boundaries, sketch_dims)

    @classmethod
    def from_variances(cls, layer_var, num_groups: int, m_avg: int, m_min: int = 32,
                       m_max: int = 1024) -> "LayerGroups":
        """Sensitivity profile: groups and sketch dims from per-layer key variances."""
        obj = cls.__new__(cls)
        obj._g = native.tq_sensitivity_profile(layer_var, num_groups, m_avg, m_min, m_max)
        return obj

    @property
    def boundaries(self):
        return [int(self._g.bound[i]) for i in range(self._g.n - 1)]

    @property
    def sketch_dims(self):
        return [int(self._g.m[i]) for i in range(self._g.n)]

    def m_for_layer(self, layer: int) -> int:
        return native.tq_m_for_layer(self._g, layer)


def key_variance(K: torch.Tensor, workspace: Optional[torch.Tensor] = None) -> float:
    """Population variance of every entry of one layer's calibration keys
    (tq_key_moments, one streaming pass on the device; waits for the result)."""
    out = torch.empty(2, dtype=torch.float64, device=K.device)
    if workspace is None:
        workspace = torch.empty(native.tq_key_moments_workspace_bytes(), dtype=torch.uint8,
                                device=K.device)
    native.tq_key_moments(K, out, workspace)
    return float(out[1].item())


class CompressedKVCache:
    """A packed cache of B x Hkv sequences plus its full-precision ring."""

    def __init__(self, B, Hkv, d, b1, m, vbits, group, W, capacity, dtype=torch.bfloat16,
                 device="cuda", structured: bool = False):
        """structured: the projections come from Projections(..., structured=True);
        the rotations on CUDA cores then run as fast Walsh-Hadamard transforms."""
        rot = native.TQ_ROTATION_HADAMARD if structured else native.TQ_ROTATION_DENSE
        self.desc = native.make_desc(B, Hkv, d, b1, m, vbits, group, W, capacity, dtype, rot)
        self.dtype = dtype
        nbytes = native.tq_cache_bytes(self.desc)
        if nbytes == 0:
            native.tq_cache_layout(self.desc)      # raises with the reason
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.state = native.tq_cache()
        native.tq_cache_init(self.state, self.desc, self.buffer)
        self._ws = None

    @property
    def n_total(self) -> int:
        return self.state.n_total

    @property
    def n_comp(self) -> int:
        return native.lib.tq_cache_compressed_tokens(self.state)

    @property
    def n_ring(self) -> int:
        return native.lib.tq_cache_ring_tokens(self.state)

    def append(self, K: torch.Tensor, V: torch.Tensor, proj: Projections, cb: Optional[Codebook]):
        native.tq_append(self.state, K, V, proj.Pi, proj.T,
                         cb.centroids if cb is not None else None,
                         cb.boundaries if cb is not None else None)

    def workspace(self, Hq: int, num_splits: int = 0) -> torch.Tensor:
        need = native.tq_decode_workspace_bytes(self.state, Hq, num_splits)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.buffer.device)
        return self._ws

    def decode_step(self, K: torch.Tensor, V: torch.Tensor, Q: torch.Tensor, proj: Projections,
                    cb: Optional[Codebook], softmax_scale: Optional[float] = None,
                    want_logits: bool = False, num_splits: int = 0,
                    out: Optional[torch.Tensor] = None):
        """append(K, V) then decode(Q) as one call (fused when the shapes allow)."""
        B, Hq, d = Q.shape
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
        out = torch.empty_like(Q) if out is None else out
        logits = None
        if want_logits:        # compressed + ring tokens after the append
            logits = torch.empty(B, Hq, self.n_total + K.shape[2], dtype=torch.float32,
                                 device=Q.device)
        ws = self.workspace(Hq, num_splits)
        native.tq_decode_step(self.state, K, V, Q, scale, proj.Pi, proj.S, proj.T,
                              cb.centroids if cb is not None else None,
                              cb.boundaries if cb is not None else None, out, logits, num_splits, ws)
        return (out, logits) if want_logits else out

    def prefill(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, proj: Projections,
                cb: Optional[Codebook], softmax_scale: Optional[float] = None, num_splits: int = 0,
                out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
        """Attention of a chunk of n new tokens before it is appended: Q [B, n, Hq, d]
        (token-major), K, V [B, Hkv, n, d]; query i sees the history, the ring and
        chunk tokens 0..i.  The cache is unchanged (call append(K, V) afterwards)."""
        B, n, Hq, d = Q.shape
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
        out = torch.empty_like(Q) if out is None else out
        if workspace is None:
            need = native.tq_prefill_workspace_bytes(self.state, Hq, n, num_splits)
            workspace = torch.empty(need, dtype=torch.uint8, device=self.buffer.device)
        native.tq_prefill_attention(self.state, Q, K, V, scale, proj.Pi, proj.S,
                                    cb.centroids if cb is not None else None, out, num_splits,
                                    workspace)
        return out

    def decode_partials(self, Q: torch.Tensor, proj: Projections, cb: Optional[Codebook],
                        softmax_scale: Optional[float] = None, num_splits: int = 0,
                        workspace: Optional[torch.Tensor] = None):
        """This cache's share of a context-sharded decode: query preparation and the
        split partials, not merged.  Returns (part_ml [B*Hq, S, 2], part_o
        [B*Hq, S, d]), float32 views into the workspace (valid until it is reused)."""
        B, Hq, d = Q.shape
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
        ws = self.workspace(Hq, num_splits) if workspace is None else workspace
        cent = cb.centroids if cb is not None else None
        native.tq_decode_prep(self.state, Q, scale, proj.Pi, proj.S, cent, num_splits, ws)
        native.tq_decode_partial(self.state, Hq, scale, cent, None, num_splits, ws)
        return native.tq_decode_partials_view(self.state, Hq, num_splits, ws)

    def decode(self, Q: torch.Tensor, proj: Projections, cb: Optional[Codebook],
               softmax_scale: Optional[float] = None, want_logits: bool = False,
               num_splits: int = 0, out: Optional[torch.Tensor] = None):
        B, Hq, d = Q.shape
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
        out = torch.empty_like(Q) if out is None else out
        logits = None
        if want_logits:
            logits = torch.empty(B, Hq, self.n_comp + self.n_ring, dtype=torch.float32, device=Q.device)
        ws = self.workspace(Hq, num_splits)
        native.tq_decode_attention(self.state, Q, scale, proj.Pi, proj.S,
                                   cb.centroids if cb is not None else None, out, logits,
                                   num_splits, ws)
        return (out, logits) if want_logits else out


# ----------------------------------------------------------------------------- sharded context
def stack_partials(parts, slots: int):
    """Split partials of several context shards side by side: parts = [(part_ml
    [rows, S_i, 2], part_o [rows, S_i, d]), ...] with S_i <= slots; a shard with
    fewer splits is padded with empty slots (m = -inf, l = 0, o = 0).  Returns
    (part_ml [rows, R * slots, 2], part_o [rows, R * slots, d]), contiguous."""
    mls, os_ = [], []
    for ml, o in parts:
        rows, s, d = o.shape
        if s > slots:
            raise ValueError(f"a shard has {s} splits, more than slots={slots}")
        pm = torch.zeros(rows, slots, 2, dtype=torch.float32, device=ml.device)
        pm[:, :, 0] = float("-inf")
        pm[:, :s] = ml
        po = torch.zeros(rows, slots, d, dtype=torch.float32, device=o.device)
        po[:, :s] = o
        mls.append(pm)
        os_.append(po)
    return torch.cat(mls, dim=1).contiguous(), torch.cat(os_, dim=1).contiguous()


def gather_partials(part_ml: torch.Tensor, part_o: torch.Tensor, slots: int, group=None):
    """All-gather every rank's split partials of one decode (each rank holds one shard
    of the context) and stack them as ``stack_partials`` does.  Every rank passes
    the same ``slots`` (at least its own split count)."""
    import torch.distributed as dist
    ml, o = stack_partials([(part_ml, part_o)], slots)
    R = dist.get_world_size(group)
    mls = [torch.empty_like(ml) for _ in range(R)]
    os_ = [torch.empty_like(o) for _ in range(R)]
    dist.all_gather(mls, ml, group=group)
    dist.all_gather(os_, o, group=group)
    return torch.cat(mls, dim=1).contiguous(), torch.cat(os_, dim=1).contiguous()


def merge_partials(part_ml: torch.Tensor, part_o: torch.Tensor, out: torch.Tensor) -> torch.Tensor:
    """out [rows, d] (any float dtype): the softmax merge of the slots of each row."""
    native.tq_merge_partials(part_ml, part_o, out)
    return out
