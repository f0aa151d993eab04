"""The generation loop's decode step captured in CUDA graphs and replayed per token.

A decode step is three launches: the fused QK-norm / RoPE / append of the new
token (``gqa_rope_append``), then the split decode over the cache and its merge
(``gqa_decode``).  At small batch each runs for a few microseconds, so issuing
them one by one from the host costs more than running them; the KV-cache loop
of page "750美元从零训练3个LLM：一位开发者的实战复盘" (section "V3：扩容与推理优化":
a prompt followed by 100 generated tokens, each token attending to the cached
keys and values) is then launch-bound.  Here the step is captured once, with
every buffer fixed: the new token's q, k and v, the output, the decode
workspace and a status word.  The per-sequence cache lengths ping-pong between
two device vectors -- the append reads one as the new token's position and
writes the other (length + 1), which the decode then reads -- so two graphs,
one for each direction, cover every step, and no host value changes between
replays.  The decode's grid covers ``max_len`` cache slots (default: the whole
capacity); the CTAs past a sequence's current length exit at once.
"""
from __future__ import annotations

import torch

from . import _lib


class DecodeGraph:
    """Replays one decode step per call of :meth:`step`.

    Write the new token's projections into ``q`` [B, Hq, D], ``k`` and ``v``
    [B, Hkv, D] (bfloat16), call :meth:`step`, and read ``out`` [B, Hq, D].
    ``lens`` (int32 [B], on the cache's device) are the cached lengths before
    the first step; :attr:`lens` is the current length vector.  The caches are
    updated in place, exactly as by the eager calls.  Device errors are OR-ed
    into ``status``.
    """

    def __init__(self, k_cache, v_cache, lens, Hq, max_len=None, qk_norm=False, eps=1e-6,
                 rope_base=10000.0, scaling=None, scale=0.0):
        if not (isinstance(k_cache, torch.Tensor) and k_cache.is_cuda):
            raise ValueError("k_cache must be a CUDA tensor (no CPU path exists)")
        B, Hkv, Lmax, D = k_cache.shape
        dev = k_cache.device
        self.max_len = Lmax if max_len is None else int(max_len)
        bf = torch.bfloat16
        self.q = torch.zeros(B, Hq, D, dtype=bf, device=dev)
        self.k = torch.zeros(B, Hkv, D, dtype=bf, device=dev)
        self.v = torch.zeros(B, Hkv, D, dtype=bf, device=dev)
        self.out = torch.zeros(B, Hq, D, dtype=bf, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self._lens = [lens.to(device=dev, dtype=torch.int32).clone(),
                      lens.to(device=dev, dtype=torch.int32).clone()]
        self._workspace = _lib.decode_workspace(B, Hq, D, self.max_len, dev)
        rope = dict(qk_norm=qk_norm, eps=eps, rope_base=rope_base, scaling=scaling)

        def one_step(a, b):
            _lib.gqa_rope_append(self.q, self.k, self.v, k_cache, v_cache, pos0=self._lens[a],
                                 new_len=self._lens[b], status=self.status, **rope)
            _lib.gqa_decode(self.q, k_cache, v_cache, self._lens[b], self.max_len, out=self.out,
                            workspace=self._workspace, scale=scale, status=self.status)

        # One eager step first, on a side stream, so that every first-use setup
        # (kernel attributes, the library load) happens outside the capture.  It
        # writes only the cache slot at each sequence's current length -- the
        # slot the first real step overwrites -- and the second length vector.
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            one_step(0, 1)
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        self.status.zero_()
        self._graphs = []
        for a, b in ((0, 1), (1, 0)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                one_step(a, b)
            self._graphs.append(g)
        self._cur = 0           # index of the length vector that holds the current lengths

    @property
    def lens(self) -> torch.Tensor:
        return self._lens[self._cur]

    def step(self) -> torch.Tensor:
        """Append the token in q, k, v at the current lengths and decode it."""
        self._graphs[self._cur].replay()
        self._cur ^= 1
        return self.out
