"""The split model the selection describes: top-K layers in 16 bits, the rest in NF4 + DQ.

arxivdaily 2608.23816, "English abstract": a single sweep over the weights orders the layers
by their NF4 error, and the highest-error ones stay in 16 bits while a byte budget allows, so
training never has to rebuild them.  "QLoRA", "How It Works": every other layer is held as
4-bit NF4 with 8-bit-encoded block scales, and its 16-bit values are rebuilt whenever a pass
needs them.

:func:`materialize` runs the fused pass over every layer (which writes each layer's NF4 + DQ
storage while it scores it), selects on the device, then keeps per layer exactly one copy:
the 16-bit tensor for a kept layer, the NF4 storage for the others.  The memory report
counts the bytes the model holds; its ``extra_bytes`` (what the kept layers cost on top of an
all-NF4 model) is the quantity the budget bounds.  All arithmetic runs in libaqnf4's kernels;
this module only allocates, sequences the calls and does the byte accounting.
"""
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

from . import aqnf4


@dataclass
class SplitLayer:
    index: int
    kind: str                         # "fp16" (kept in 16 bits) or "nf4"
    shape: tuple
    dtype: torch.dtype                # the layer's 16-bit format
    rel_err: float                    # the score the selection ranked
    weight: Optional[torch.Tensor]    # kept layers: the caller's 16-bit tensor
    nf4: Optional[aqnf4.NF4Storage]   # other layers: packed codes + DQ constants

    @property
    def numel(self) -> int:
        n = 1
        for d in self.shape:
            n *= d
        return n

    def held_bytes(self) -> int:
        if self.kind == "fp16":
            return self.weight.numel() * self.weight.element_size()
        return nf4_bytes(self.nf4)


def nf4_bytes(st: aqnf4.NF4Storage) -> int:
    return sum(t.numel() * t.element_size() for t in (st.packed, st.codes8, st.scales))


class SplitModel:
    """``layers`` in input order; ``ranking`` is the selection's whole ranking and ``kept``
    its first k entries (the layers held in 16 bits)."""

    def __init__(self, layers: List[SplitLayer], ranking: List[int], kept: List[int],
                 budget_bytes: int):
        self.layers = layers
        self.ranking = ranking
        self.kept = kept
        self.budget_bytes = budget_bytes

    def weight(self, i: int, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Layer i as 16-bit weights: the kept tensor itself, or the NF4 storage dequantized
        into ``out`` (allocated when None) on the given stream."""
        L = self.layers[i]
        if L.kind == "fp16":
            return L.weight
        st = L.nf4
        if out is None:
            out = torch.empty(L.shape, dtype=L.dtype, device=st.packed.device)
        aqnf4.aqnf4_dequantize(st.packed, st.codes8, st.scales, None, L.numel, out, stream)
        return out

    def linear_path(self, i: int, x_dtype: torch.dtype) -> str:
        """Which path linear(i, x) takes for an x of the given dtype:
        "cublas-16bit" (a kept layer), "fused-nf4" (the fused NF4-dequant tensor-core GEMM), or
        "dequantize+cublas" (an NF4 layer whose K is not a multiple of 64, or an x whose 16-bit
        format differs from the layer's: the layer is dequantized, x converted to the layer's
        format, and cuBLAS multiplies)."""
        L = self.layers[i]
        if L.kind == "fp16":
            return "cublas-16bit"
        if len(L.shape) != 2 or L.shape[1] % 64 != 0 or x_dtype != L.dtype:
            return "dequantize+cublas"
        return "fused-nf4"

    def linear(self, i: int, x: torch.Tensor, out_dtype: Optional[torch.dtype] = None,
               stream=None) -> torch.Tensor:
        """The forward product of layer i, y = x w^T, for x (M x K): cuBLAS on the kept 16-bit
        weights, or the fused NF4-dequant tensor-core GEMM (aqnf4_nf4_linear) on the NF4 + DQ
        storage.  A layer whose K is not a multiple of 64 (rows would not be whole NF4 blocks),
        or an x in the other 16-bit format, is dequantized first and multiplied by cuBLAS with
        x converted to the layer's format; linear_path(i, x.dtype) names the path taken."""
        L = self.layers[i]
        if len(L.shape) != 2:
            raise ValueError("linear: the layer is not a matrix")
        N, K = L.shape
        out_dtype = out_dtype or x.dtype
        path = self.linear_path(i, x.dtype)

        def dense(w16):  # cuBLAS; a float32 result is summed in binary32 without 16-bit rounding
            if out_dtype == torch.float32:
                return torch.matmul(x.to(L.dtype).float(), w16.float().t())
            return torch.matmul(x.to(L.dtype), w16.t()).to(out_dtype)

        if path == "cublas-16bit":
            return dense(L.weight)
        if path == "dequantize+cublas":
            return dense(self.weight(i, stream=stream))
        M = x.shape[0]
        y = torch.empty((M, N), dtype=out_dtype if out_dtype == torch.float32 else x.dtype,
                        device=x.device)
        st = L.nf4
        aqnf4.aqnf4_nf4_linear(x.contiguous(), st.packed, st.codes8, st.scales, N, y,
                               stream=stream)
        return y.to(out_dtype)

    def memory_report(self) -> dict:
        fp16 = sum(L.held_bytes() for L in self.layers if L.kind == "fp16")
        nf4 = sum(L.held_bytes() for L in self.layers if L.kind == "nf4")
        all_nf4 = sum(nf4_storage_bytes(L.numel) for L in self.layers)
        extra = fp16 + nf4 - all_nf4
        return {"layers": len(self.layers), "fp16_layers": len(self.kept),
                "fp16_bytes": fp16, "nf4_bytes": nf4, "total_bytes": fp16 + nf4,
                "all_nf4_bytes": all_nf4, "extra_bytes": extra,
                "budget_bytes": self.budget_bytes, "within_budget": extra <= self.budget_bytes}


def nf4_storage_bytes(n: int) -> int:
    """Bytes of one layer's NF4 + DQ storage: ceil(n/2) + ceil(n/64) + 4 ceil(ceil(n/64)/256)."""
    return 2 * n - aqnf4.aqnf4_cost_bytes(n)


def materialize(weights: Sequence[torch.Tensor], budget_bytes: int, k_cap: int = -1,
                dq_score: bool = False, stream=None) -> SplitModel:
    """Score every layer, select the top-K under ``budget_bytes`` (and ``k_cap``), and return
    the split model.  ``weights`` are 16-bit device tensors (bf16 or fp16, any shape).  The
    model keeps references to the kept layers' tensors only; the caller may drop its own
    references to the others.  ``dq_score`` ranks by the error of the double-quantized model
    (AQNF4_SCORE_DQ_ABSMAX)."""
    weights = list(weights)
    if not weights:
        raise ValueError("materialize: no layers")
    dev = weights[0].device
    flat = [w.reshape(-1) for w in weights]
    stor = [aqnf4.NF4Storage(w.numel(), dev) for w in flat]
    _, _, rel = aqnf4.score_layers(flat, stor, stream=stream, dq_score=dq_score)
    cost = torch.tensor([aqnf4.aqnf4_cost_bytes(w.numel()) for w in flat], dtype=torch.int64,
                        device=dev)
    sel, k = aqnf4.select_topk(rel, cost, budget_bytes, k_cap, stream=stream)
    if stream is not None:
        stream.synchronize()
    k = int(k.item())
    ranking = sel.tolist()
    kept = ranking[:k]
    keep = set(kept)
    rel_h = rel.tolist()
    layers = []
    for i, w in enumerate(weights):
        if i in keep:
            layers.append(SplitLayer(i, "fp16", tuple(w.shape), w.dtype, rel_h[i], w, None))
        else:
            layers.append(SplitLayer(i, "nf4", tuple(w.shape), w.dtype, rel_h[i], None, stor[i]))
    del stor
    return SplitModel(layers, ranking, kept, budget_bytes)


__all__ = ["SplitLayer", "SplitModel", "materialize", "nf4_bytes", "nf4_storage_bytes"]
