"""Device memory and streams for one context of the C ABI.  PyTorch only
allocates (workspace, slot arena) and provides the two CUDA streams; every
step of the layer runs inside libmoeoffload.so.

Buffers passed to the forward calls must be ready before the call: the
library's work is ordered on its own compute stream, so a caller that filled
them on another stream synchronises first (or makes the compute stream wait)."""
from __future__ import annotations

import torch

from . import abi


class LayerStack:
    """One moe_ctx: L layers of routed experts behind a global LRU slot cache.

    host_pool: page-locked uint8 tensor of P expert records (the pinned host pool).
    router_w: device tensor, bf16 [L, E, d] (or its uint16 bit pattern).
    shared: device uint8 tensor of L shared-expert records (abi.moe_shared_record_bytes each), or None.
    """

    def __init__(self, dims: abi.moe_dims, host_pool: torch.Tensor, router_w: torch.Tensor,
                 shared: torch.Tensor | None, num_slots: int, *, prefetch: bool = False,
                 static_split: bool = False, shard: tuple[int, int] = (0, 1),
                 device: str | torch.device = "cuda"):
        if not torch.cuda.is_available():
            raise RuntimeError("LayerStack needs a CUDA device")
        self.dims = dims
        self.device = torch.device(device)
        self.num_slots = num_slots
        self.record_bytes = abi.moe_record_bytes(dims)
        self.ws = torch.empty(abi.moe_workspace_bytes(dims), dtype=torch.uint8, device=self.device)
        self.arena = torch.empty(abi.moe_arena_bytes(dims, num_slots), dtype=torch.uint8,
                                 device=self.device)
        self.compute = torch.cuda.Stream(device=self.device)
        self.copy = torch.cuda.Stream(device=self.device)
        self.host_pool, self.router_w, self.shared = host_pool, router_w, shared
        torch.cuda.synchronize(self.device)
        self.ctx = abi.moe_layer_init(dims, host_pool, host_pool.numel(), router_w, shared,
                                      self.ws, self.ws.numel(), self.compute, self.copy)
        self.flags = ((abi.MOE_CACHE_PREFETCH_NEXT if prefetch else 0) |
                      (abi.MOE_CACHE_STATIC_SPLIT if static_split else 0))
        if shard != (0, 1):  # expert parallelism: this stack serves experts e % size == rank
            abi.moe_set_expert_shard(self.ctx, shard[0], shard[1])
        self.reset()

    def reset(self) -> None:
        abi.cache_configure(self.ctx, self.num_slots, self.arena, self.arena.numel(),
                            abi.MOE_CACHE_RESET | self.flags)

    def forward(self, layer: int, x: torch.Tensor, y: torch.Tensor, trace=None) -> None:
        abi.moe_layer_forward(self.ctx, layer, x, x.shape[0], y, trace)

    def forward_host(self, layer: int, x_host: torch.Tensor, y_host: torch.Tensor,
                     trace=None) -> None:
        abi.moe_layer_forward_host(self.ctx, layer, x_host, x_host.shape[0], y_host, trace)

    def synchronize(self) -> None:
        self.compute.synchronize()

    def close(self) -> None:
        if getattr(self, "ctx", None):
            abi.moe_layer_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def new_trace(capacity: int):
    """A host trace buffer for moe_layer_forward: (struct, backing array)."""
    arr = (abi.moe_cache_event * capacity)()
    tr = abi.moe_layer_trace(arr, capacity, 0)
    return tr, arr


def trace_events(tr, arr) -> list[tuple[int, int, int, int, int, int]]:
    """[(layer, expert, slot, hit, evicted_key, prefetch)] of the last call."""
    n = min(tr.count, tr.capacity)
    return [(arr[i].layer, arr[i].expert, arr[i].slot, arr[i].hit, arr[i].evicted_key,
             arr[i].prefetch) for i in range(n)]
