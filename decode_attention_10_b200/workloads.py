"""Seeded synthetic inputs for one MFA decode step.

This module only draws random numbers and lays them out; it holds none of the layer's
arithmetic. It is the one piece shared by the CUDA path's tests/benchmark and by the
float64 oracle, which both read the exact bytes produced here.

Shapes follow the Step-3 pages (bud-325 summary, "Key claims"/"Method"; redeep.blog
architecture table): hidden 7168, low-rank query 2048, 64 query heads of dimension 256,
one shared K head and one shared V head of dimension 256, context up to 65,536.

Recipe (every workload):
  * generator: ``torch.Generator`` on the CPU, seed ``1000 + workload index`` unless given;
  * draw order: x, W_qdown, W_qup, W_k, W_v, K cache, V cache; ragged workloads draw
    their lengths first from their own generator (seed) and the rest from seed + 1;
  * x ~ N(0, 1) [B, 7168]; W_qdown [7168, 2048] ~ N(0, 1/7168); W_qup [2048, 16384]
    ~ N(0, 1/2048); W_k, W_v [7168, 256] ~ N(0, 1/7168); gamma = 1 [2048];
  * K/V cache rows ~ N(0, 1); every value is drawn in float32 and rounded to bf16
    (round to nearest even, torch's conversion);
  * FP8 workloads: the float32 N(0,1) cache values are quantized by torch's float8_e4m3fn
    conversion with one float32 scale per tensor, scale = max|value| / 448;
  * each sequence's cache has capacity = its length L_b; the decode step overwrites row
    L_b - 1 with the new token's K/V, so after the step the cache is exactly full.
"""

from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

HIDDEN = 7168
Q_RANK = 2048
N_HEADS = 64
HEAD_DIM = 256
MAX_CONTEXT = 65536

KV_BF16 = "bf16"
KV_FP8 = "fp8_e4m3"


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    batch: int
    kv_dtype: str
    context: Optional[int]  # uniform context L; None = ragged lengths U[1, MAX_CONTEXT]
    contiguous: bool = True  # one [B, L, 256] buffer per cache, else one buffer per sequence
    note: str = ""


WORKLOADS = (
    Workload(0, "mfa_decode_b1_l128_bf16", 1, KV_BF16, 128,
             note="batch 1, context 128, bf16 KV"),
    Workload(1, "mfa_decode_b32_l4096_bf16", 32, KV_BF16, 4096,
             note="batch 32, uniform context 4096, bf16 KV"),
    Workload(2, "mfa_decode_b64_l8192_bf16", 64, KV_BF16, 8192,
             note="batch 64, uniform context 8192, bf16 KV"),
    Workload(3, "mfa_decode_b128_l4096_fp8", 128, KV_FP8, 4096,
             note="batch 128, uniform context 4096, FP8 e4m3 KV, per-tensor scales"),
    Workload(4, "mfa_decode_b16_ragged64k_bf16", 16, KV_BF16, None, contiguous=False,
             note="batch 16, lengths U[1, 65536], bf16 KV in per-sequence buffers"),
)


def workload(index_or_name) -> Workload:
    for w in WORKLOADS:
        if w.index == index_or_name or w.name == index_or_name:
            return w
    raise KeyError(index_or_name)


@dataclass
class Inputs:
    """Host (CPU) tensors of one decode step. Cache tensors hold the stored codes:
    torch.bfloat16 or torch.float8_e4m3fn, one [cap_b, 256] tensor per sequence (views into
    one [B, L, 256] buffer for contiguous workloads)."""
    x: torch.Tensor
    w_qdown: torch.Tensor
    gamma: torch.Tensor
    w_qup: torch.Tensor
    w_k: torch.Tensor
    w_v: torch.Tensor
    k_cache: list
    v_cache: list
    seq_lens: torch.Tensor  # int32 [B]: positions attended after the append
    kv_dtype: str
    k_scale: float = 1.0
    v_scale: float = 1.0
    k_buffer: Optional[torch.Tensor] = None  # the [B, L, 256] buffer of contiguous caches
    v_buffer: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.x.shape[0])


def _randn(g, *shape, std=1.0):
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def _e4m3_scale(tensors) -> float:
    """One float32 scale per tensor: max|value| / 448 (448 = largest finite e4m3)."""
    amax = max(float(t.abs().max()) for t in tensors)
    if amax == 0:
        return 1.0
    return float(torch.tensor(amax / 448.0, dtype=torch.float32))


def generate(seq_lens: Sequence[int], kv_dtype: str = KV_BF16, seed: int = 0,
             contiguous: Optional[bool] = None, capacity: Optional[Sequence[int]] = None,
             x_scale: float = 1.0) -> Inputs:
    """Draw the inputs of one decode step for the given per-sequence lengths.

    ``capacity[b] >= seq_lens[b]`` rows are allocated per sequence (default: the length).
    ``contiguous`` (default: all lengths equal and capacities equal) puts every sequence's
    cache in one [B, cap, 256] buffer."""
    lens = [int(n) for n in seq_lens]
    bsz = len(lens)
    caps = list(lens) if capacity is None else [int(c) for c in capacity]
    if any(c < n for c, n in zip(caps, lens)):
        raise ValueError("capacity below length")
    if contiguous is None:
        contiguous = len(set(caps)) == 1
    g = torch.Generator().manual_seed(int(seed))
    x = _randn(g, bsz, HIDDEN, std=x_scale).to(torch.bfloat16)
    w_qdown = _randn(g, HIDDEN, Q_RANK, std=HIDDEN ** -0.5).to(torch.bfloat16)
    w_qup = _randn(g, Q_RANK, N_HEADS * HEAD_DIM, std=Q_RANK ** -0.5).to(torch.bfloat16)
    w_k = _randn(g, HIDDEN, HEAD_DIM, std=HIDDEN ** -0.5).to(torch.bfloat16)
    w_v = _randn(g, HIDDEN, HEAD_DIM, std=HIDDEN ** -0.5).to(torch.bfloat16)
    gamma = torch.ones(Q_RANK, dtype=torch.bfloat16)

    def draw_cache():
        if contiguous:
            return [_randn(g, bsz, caps[0], HEAD_DIM)]
        return [_randn(g, c, HEAD_DIM) for c in caps]

    k_vals = draw_cache()
    v_vals = draw_cache()
    k_scale = v_scale = 1.0
    if kv_dtype == KV_BF16:
        k_store = [t.to(torch.bfloat16) for t in k_vals]
        v_store = [t.to(torch.bfloat16) for t in v_vals]
    elif kv_dtype == KV_FP8:
        k_scale = _e4m3_scale(k_vals)
        v_scale = _e4m3_scale(v_vals)
        k_store = [(t / k_scale).to(torch.float8_e4m3fn) for t in k_vals]
        v_store = [(t / v_scale).to(torch.float8_e4m3fn) for t in v_vals]
    else:
        raise ValueError(kv_dtype)
    del k_vals, v_vals
    if contiguous:
        k_buf, v_buf = k_store[0], v_store[0]
        k_cache = [k_buf[b] for b in range(bsz)]
        v_cache = [v_buf[b] for b in range(bsz)]
    else:
        k_buf = v_buf = None
        k_cache, v_cache = k_store, v_store
    return Inputs(x=x, w_qdown=w_qdown, gamma=gamma, w_qup=w_qup, w_k=w_k, w_v=w_v,
                  k_cache=k_cache, v_cache=v_cache,
                  seq_lens=torch.tensor(lens, dtype=torch.int32), kv_dtype=kv_dtype,
                  k_scale=float(k_scale), v_scale=float(v_scale), k_buffer=k_buf,
                  v_buffer=v_buf, meta=dict(seed=int(seed), capacity=caps))


def generate_w_o(seed: int) -> torch.Tensor:
    """The output projection W_o [16384, 7168] of one layer, bf16 ~ N(0, 1/16384) (the same
    fan-in scaling as the other projections)."""
    g = torch.Generator().manual_seed(int(seed))
    width = N_HEADS * HEAD_DIM
    return _randn(g, width, HIDDEN, std=width ** -0.5).to(torch.bfloat16)


def generate_layer_on_device(seq_lens: Sequence[int], kv_dtype: str, seed: int, device,
                             contiguous: bool = True) -> dict:
    """One layer's weights (W_qdown, gamma, W_qup, W_k, W_v, W_o) and KV cache drawn on the
    device with the distributions of ``generate`` and ``generate_w_o``, for stacks of many
    layers whose tensors would take minutes to draw on the host. Returns a dict with those
    tensors, k_cache / v_cache (per-sequence views) and k_scale / v_scale."""
    lens = [int(n) for n in seq_lens]
    bsz = len(lens)
    g = torch.Generator(device=device).manual_seed(int(seed))

    def randn(*shape, std=1.0):
        t = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
        return t.mul_(std) if std != 1.0 else t

    width = N_HEADS * HEAD_DIM
    d = dict(w_qdown=randn(HIDDEN, Q_RANK, std=HIDDEN ** -0.5).to(torch.bfloat16),
             w_qup=randn(Q_RANK, width, std=Q_RANK ** -0.5).to(torch.bfloat16),
             w_k=randn(HIDDEN, HEAD_DIM, std=HIDDEN ** -0.5).to(torch.bfloat16),
             w_v=randn(HIDDEN, HEAD_DIM, std=HIDDEN ** -0.5).to(torch.bfloat16),
             w_o=randn(width, HIDDEN, std=width ** -0.5).to(torch.bfloat16),
             gamma=torch.ones(Q_RANK, dtype=torch.bfloat16, device=device))
    for name in ("k", "v"):
        if contiguous:
            vals = [randn(bsz, max(lens), HEAD_DIM)]
        else:
            vals = [randn(n, HEAD_DIM) for n in lens]
        if kv_dtype == KV_BF16:
            scale = 1.0
            store = [t.to(torch.bfloat16) for t in vals]
        else:
            amax = max(float(t.abs().max()) for t in vals)
            scale = float(torch.tensor(amax / 448.0, dtype=torch.float32)) if amax else 1.0
            store = [(t / scale).to(torch.float8_e4m3fn) for t in vals]
        del vals
        d[name + "_scale"] = scale
        d[name + "_buffer"] = store
        d[name + "_cache"] = [store[0][b] for b in range(bsz)] if contiguous else store
    return d


def quantize_w8(w: torch.Tensor, block: int = 128):
    """A bf16 weight [in, out] drawn by ``generate``, stored as block FP8 in the checkpoints'
    order: e4m3 codes [out, in] (uint8) and one float32 scale per block x block tile (its
    largest |w| / 448; 1 for an all-zero tile), the values w / scale rounded to nearest even
    and kept within +-448. Returns (codes, scales) on w's device."""
    wt = w.t().float()
    o, i = wt.shape
    bo, bi = -(-o // block), -(-i // block)
    pad = torch.zeros(bo * block, bi * block, dtype=torch.float32, device=w.device)
    pad[:o, :i] = wt
    tiles = pad.view(bo, block, bi, block)
    amax = tiles.abs().amax(dim=(1, 3))
    scales = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).float()
    q = (tiles / scales[:, None, :, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    codes = q.view(bo * block, bi * block)[:o, :i].contiguous().view(torch.uint8)
    return codes, scales.contiguous()


def to_paged(k_cache: Sequence[torch.Tensor], v_cache: Sequence[torch.Tensor], page_size: int,
             seed: int, spare_pages: int = 0, shuffle: bool = True):
    """The per-sequence caches ([capacity_b, 256] tensors, on any device) copied into K and V
    page pools [num_pages, page_size, 256] at shuffled pool positions (a serving engine's
    page allocator hands pages out in no particular order). Rows of a sequence's last page
    past its capacity are zero; ``shuffle=False`` lays the pages out in sequence order
    instead. Returns (k_pool, v_pool, page_table int32 [B, max_pages] on
    the caches' device, pages per sequence)."""
    caps = [int(t.shape[0]) for t in k_cache]
    need = [-(-c // page_size) for c in caps]
    total = sum(need) + int(spare_pages)
    g = torch.Generator().manual_seed(int(seed))
    order = torch.randperm(total, generator=g) if shuffle else torch.arange(total)
    table = torch.zeros(len(caps), max(need), dtype=torch.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = order[at:at + n].to(torch.int32)
        at += n
    dev = k_cache[0].device
    pools = []
    for cache in (k_cache, v_cache):
        pool = torch.zeros(total, page_size, HEAD_DIM, dtype=cache[0].dtype, device=dev)
        flat = pool.view(-1) if cache[0].element_size() == 2 else pool.view(torch.uint8).view(-1)
        for b, t in enumerate(cache):
            rows = t.reshape(-1) if t.element_size() == 2 else t.view(torch.uint8).reshape(-1)
            # page p of sequence b: rows [p * page_size, (p + 1) * page_size) of its cache
            for p in range(need[b]):
                lo = p * page_size * HEAD_DIM
                hi = min(caps[b] * HEAD_DIM, lo + page_size * HEAD_DIM)
                base = int(table[b, p]) * page_size * HEAD_DIM
                flat[base:base + hi - lo].copy_(rows[lo:hi])
        pools.append(pool)
    return pools[0], pools[1], table.to(dev), need


def ragged_lengths(batch: int, seed: int) -> list:
    """Per-sequence lengths drawn uniform in [1, 65536] -- the first draw of the seed."""
    g = torch.Generator().manual_seed(int(seed))
    return [int(n) for n in torch.randint(1, MAX_CONTEXT + 1, (batch,), generator=g)]


def workload_lens(w: Workload, seed: Optional[int] = None) -> list:
    """The per-sequence lengths of a named workload, without drawing its tensors."""
    seed = 1000 + w.index if seed is None else int(seed)
    return ragged_lengths(w.batch, seed) if w.context is None else [w.context] * w.batch


def generate_workload(w: Workload, seed: Optional[int] = None) -> Inputs:
    """Inputs of one of the named workloads (seed defaults to 1000 + index)."""
    seed = 1000 + w.index if seed is None else int(seed)
    if w.context is None:
        lens = ragged_lengths(w.batch, seed)
        inp = generate(lens, w.kv_dtype, seed=seed + 1, contiguous=w.contiguous)
    else:
        inp = generate([w.context] * w.batch, w.kv_dtype, seed=seed,
                       contiguous=w.contiguous)
    inp.meta["workload"] = w.name
    return inp
