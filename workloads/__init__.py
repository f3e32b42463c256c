"""Seeded synthetic decode workloads shaped like the vLLM / PagedAttention pages.

This module is shared by the tests, the benchmark and the oracle checks, and
holds none of the method's arithmetic: it only draws context lengths, free-list
orders and random K/V/q contents, and writes down the block-manager operations
(add / fork / append / release) that build each batch.  Each side (CUDA library
or oracle) replays those operations on its own allocator, writes the K/V with
its own append routine and computes attention on its own cache.

Workloads (stand-ins for the ShareGPT / Alpaca-shaped OPT and LLaMA serving
workloads of "구현과 실험 환경" on the supersilo.blog vLLM summary, which are
not available here; shapes follow the public model configurations):

  tiny         8 seqs, context ~ U[1,64], Hq=Hkv=4, D=64, block 16, 64 blocks in
               a permuted pool, fp32 N(0,1), scale 1/8
  opt13b       64 seqs, Hq=Hkv=40, D=128, block 16, fp16 N(0,1), context
               lognormal(median 600, sigma 0.5) clipped to [16,2048], pool 20,000
  llama13b_ps  16 prompts x 6 samples, Hq=Hkv=40, D=128, bf16, prompt ~ U[512,1024]
               shared through forked (refcounted) blocks, 1..256 divergent tokens
  gqa70b       256 seqs, Hq=64, Hkv=8, D=128, bf16, block 16, context ~ U[256,4096]
               (no partition length is given: the library's automatic one)
  long_prefix  128 requests forked from one 4096-token prefix (same physical
               blocks) plus a unique suffix ~ U[1,28672]; Hq=32, Hkv=8, D=128,
               bf16, block 8/16/32, split-K partitions of 512 tokens

Any workload can keep its cache as E4M3 codes (``fp8(spec)``, named with an
``_fp8`` suffix): K/V are drawn as usual in the workload's dtype (which stays
the query / output type) and quantised on append with per-cache scales
k_scale = 0.0123 and v_scale = 0.0171 (N(0,1) contents span about +-5.5, i.e.
codes up to about 450 / 320 before saturation; the values are not powers of
two, so the fp32 quotient really rounds).

Choices the workload descriptions leave open (stated here and in the design
notes): the lognormal sigma 0.5; integer-uniform prompt, divergent and suffix
lengths; pool sizes of 1.25x the blocks needed (rounded up) where no pool is
given; q drawn like K/V, in the cache dtype; sample 0 of each prompt is the
prompt sequence itself and samples 1..5 are forks of it.

The "step" of a workload is the last group of appends: one new token per
sequence for tiny / opt13b / gqa70b / long_prefix, and every sample's divergent
tokens (with their copy-on-write of the shared prompt tail) for llama13b_ps.
Context lengths include the tokens the step appends.
"""
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

DTYPE_CODES = {"f32": 0, "f16": 1, "bf16": 2, "e4m3": 3}
DTYPE_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}
FP8_K_SCALE, FP8_V_SCALE = 0.0123, 0.0171


@dataclass(frozen=True)
class Spec:
    name: str
    dtype: str
    Hq: int
    Hkv: int
    D: int
    block_size: int
    kind: str                       # 'independent' | 'parallel_sampling' | 'shared_prefix'
    num_seqs: int                   # decode batch size B
    seed: int
    num_blocks: Optional[int] = None  # pool size; None = 1.25x what the script needs
    scale: Optional[float] = None     # None = 1/sqrt(D)
    partition_size: int = 512       # 0 = the library's automatic choice
    # independent
    ctx_dist: str = "uniform"       # 'uniform' | 'lognormal' | 'explicit'
    ctx_list: Tuple[int, ...] = ()  # explicit context lengths (num_seqs of them)
    ctx_lo: int = 1
    ctx_hi: int = 64
    ctx_median: float = 600.0
    ctx_sigma: float = 0.5
    # parallel sampling
    num_prompts: int = 0
    samples_per_prompt: int = 0
    prompt_lo: int = 0
    prompt_hi: int = 0
    div_lo: int = 0
    div_hi: int = 0
    # shared prefix
    prefix_len: int = 0
    suffix_lo: int = 0
    suffix_hi: int = 0
    # cache storage: "" = the dtype itself, "e4m3" = E4M3 codes with these scales
    kv_dtype: str = ""
    k_scale: float = 1.0
    v_scale: float = 1.0

    @property
    def dtype_code(self) -> int:
        return DTYPE_CODES[self.dtype]

    @property
    def esize(self) -> int:
        return DTYPE_BYTES[self.dtype]

    @property
    def kv(self) -> str:
        return self.kv_dtype or self.dtype

    @property
    def kv_code(self) -> int:
        return DTYPE_CODES[self.kv]

    @property
    def kv_esize(self) -> int:
        return DTYPE_BYTES[self.kv]

    @property
    def fp8(self) -> bool:
        return self.kv == "e4m3"

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def softmax_scale(self) -> float:
        s = self.scale if self.scale is not None else 1.0 / np.sqrt(self.D)
        return float(np.float32(s))


TINY = Spec("tiny", "f32", 4, 4, 64, 16, "independent", 8, seed=443, num_blocks=64,
            scale=1.0 / 8, ctx_dist="uniform", ctx_lo=1, ctx_hi=64)
OPT13B = Spec("opt13b", "f16", 40, 40, 128, 16, "independent", 64, seed=444,
              num_blocks=20000, ctx_dist="lognormal", ctx_median=600.0, ctx_sigma=0.5,
              ctx_lo=16, ctx_hi=2048, partition_size=0)
LLAMA13B_PS = Spec("llama13b_ps", "bf16", 40, 40, 128, 16, "parallel_sampling", 96, seed=445,
                   num_prompts=16, samples_per_prompt=6, prompt_lo=512, prompt_hi=1024,
                   div_lo=1, div_hi=256, partition_size=0)
GQA70B = Spec("gqa70b", "bf16", 64, 8, 128, 16, "independent", 256, seed=446,
              ctx_dist="uniform", ctx_lo=256, ctx_hi=4096, partition_size=0)
LONG_PREFIX = Spec("long_prefix", "bf16", 32, 8, 128, 16, "shared_prefix", 128, seed=447,
                   prefix_len=4096, suffix_lo=1, suffix_hi=28672, partition_size=512)

FULL = {s.name: s for s in (TINY, OPT13B, LLAMA13B_PS, GQA70B, LONG_PREFIX)}


def fp8(spec: Spec) -> Spec:
    """The workload with an E4M3 cache (queries and outputs keep spec.dtype)."""
    return replace(spec, name=spec.name + "_fp8", kv_dtype="e4m3",
                   k_scale=float(np.float32(FP8_K_SCALE)), v_scale=float(np.float32(FP8_V_SCALE)))


def long_prefix(block_size: int) -> Spec:
    return replace(LONG_PREFIX, name=f"long_prefix_bs{block_size}", block_size=block_size)


def small(name: str) -> Spec:
    """Scaled-down versions the oracle finishes in seconds; each still spans
    several tiles, several split-K partitions and a ragged last block."""
    if name == "tiny":
        return TINY
    if name == "opt13b":
        return replace(OPT13B, name="opt13b_small", num_seqs=12, Hq=6, Hkv=6, num_blocks=2000,
                       ctx_median=600.0, seed=1444)
    if name == "llama13b_ps":
        return replace(LLAMA13B_PS, name="llama13b_ps_small", num_prompts=3, samples_per_prompt=6,
                       num_seqs=18, Hq=4, Hkv=4, seed=1445)
    if name == "gqa70b":
        return replace(GQA70B, name="gqa70b_small", num_seqs=10, Hq=16, Hkv=2, ctx_lo=1,
                       ctx_hi=1500, seed=1446)
    if name == "long_prefix":
        return replace(LONG_PREFIX, name="long_prefix_small", num_seqs=6, Hq=8, Hkv=2,
                       prefix_len=1024, suffix_lo=1, suffix_hi=1800, seed=1447)
    raise KeyError(name)


@dataclass
class Op:
    kind: str          # 'add' | 'fork' | 'append' | 'release'
    seq: int
    arg: int = 0       # fork: child id; append: token count
    kv_id: int = -1    # append: which K/V content draw


@dataclass
class Scenario:
    spec: Spec
    num_blocks: int
    free_order: np.ndarray          # int32 permutation; the last entry is used first
    setup_ops: List[Op]
    step_ops: List[Op]
    batch: List[int]                # decode order of sequence ids
    context_lens: np.ndarray        # int32 [B], expected after the step (for sizing only)
    max_blocks: int                 # block-table row length
    max_context_len: int
    # where each sequence's tokens come from: seq id -> [(kv_id, first position,
    # count)] in position order (a fork inherits its parent's list)
    segments: Dict[int, List[Tuple[int, int, int]]] = field(default_factory=dict)
    # tokens at the start of each sequence that its family (the forks of one
    # parent) holds in common: the prompt of parallel samples, the prefix of
    # shared-prefix requests; 0 for independent sequences
    shared: Dict[int, int] = field(default_factory=dict)
    spikes: Optional["SpikePlan"] = None   # boundary-dominant contents (spike_plan)

    @property
    def B(self) -> int:
        return len(self.batch)


def _ctx_lengths(spec: Spec, rng) -> np.ndarray:
    B = spec.num_seqs
    if spec.ctx_dist == "uniform":
        return rng.integers(spec.ctx_lo, spec.ctx_hi + 1, size=B)
    if spec.ctx_dist == "lognormal":
        x = rng.lognormal(mean=np.log(spec.ctx_median), sigma=spec.ctx_sigma, size=B)
        return np.clip(np.rint(x), spec.ctx_lo, spec.ctx_hi).astype(np.int64)
    if spec.ctx_dist == "explicit":
        assert len(spec.ctx_list) == B
        return np.asarray(spec.ctx_list, dtype=np.int64)
    raise ValueError(spec.ctx_dist)


def scenario(spec: Spec) -> Scenario:
    """The block-manager script and sizes of one workload (seeded)."""
    rng = np.random.default_rng(spec.seed)
    bs = spec.block_size
    setup: List[Op] = []
    step: List[Op] = []
    kv = 0
    segs: Dict[int, List[Tuple[int, int, int]]] = {}

    def app(lst, sid, n):
        nonlocal kv
        if n > 0:
            lst.append(Op("append", sid, int(n), kv))
            seg = segs.setdefault(sid, [])
            pos = seg[-1][1] + seg[-1][2] if seg else 0
            seg.append((kv, pos, int(n)))
            kv += 1

    def fork(parent, child):
        setup.append(Op("fork", parent, child))
        segs[child] = list(segs.get(parent, []))

    shared: Dict[int, int] = {}
    if spec.kind == "independent":
        lens = _ctx_lengths(spec, rng)
        batch = list(range(spec.num_seqs))
        for sid, L in zip(batch, lens):
            setup.append(Op("add", sid))
            app(setup, sid, L - 1)
        for sid, L in zip(batch, lens):
            if L > 0:                   # an empty sequence appends nothing
                app(step, sid, 1)
        blocks_needed = max(1, int(sum(-(-int(L) // bs) for L in lens)))
    elif spec.kind == "parallel_sampling":
        P, S = spec.num_prompts, spec.samples_per_prompt
        prompts = rng.integers(spec.prompt_lo, spec.prompt_hi + 1, size=P)
        divs = rng.integers(spec.div_lo, spec.div_hi + 1, size=(P, S))
        batch, lens = [], []
        for p in range(P):
            root = p * S
            setup.append(Op("add", root))
            app(setup, root, prompts[p])
            for s in range(1, S):
                fork(root, root + s)
            for s in range(S):
                shared[root + s] = int(prompts[p])
        for p in range(P):
            for s in range(S):
                sid = p * S + s
                batch.append(sid)
                app(step, sid, divs[p, s])
                lens.append(int(prompts[p] + divs[p, s]))
        lens = np.array(lens)
        blocks_needed = int(sum(-(-int(x) // bs) for x in prompts)) + \
            int(sum(-(-int(prompts[p] + divs[p, s]) // bs) - int(prompts[p]) // bs
                    for p in range(P) for s in range(S)))
    elif spec.kind == "shared_prefix":
        root = 1_000_000
        setup.append(Op("add", root))
        app(setup, root, spec.prefix_len)
        suffix = rng.integers(spec.suffix_lo, spec.suffix_hi + 1, size=spec.num_seqs)
        batch = list(range(spec.num_seqs))
        for sid in batch:
            fork(root, sid)
            shared[sid] = int(spec.prefix_len)
        setup.append(Op("release", root))
        for sid, sfx in zip(batch, suffix):
            app(setup, sid, sfx - 1)
        for sid in batch:
            app(step, sid, 1)
        lens = spec.prefix_len + suffix
        blocks_needed = -(-spec.prefix_len // bs) + int(sum(-(-int(x) // bs) for x in suffix))
    else:
        raise ValueError(spec.kind)

    nb = spec.num_blocks if spec.num_blocks is not None else int(np.ceil(1.25 * blocks_needed))
    free_order = rng.permutation(nb).astype(np.int32)
    lens = np.asarray(lens, dtype=np.int32)
    max_ctx = int(lens.max()) if lens.size else 0
    max_blocks = max(1, -(-max_ctx // bs))
    return Scenario(spec, nb, free_order, setup, step, batch, lens, max_blocks, max_ctx,
                    segments={sid: segs.get(sid, []) for sid in batch},
                    shared={sid: shared.get(sid, 0) for sid in batch})


# ---------------------------------------------------------------------------
# Random contents.  Drawn with torch so large pools can be filled on the GPU;
# a draw is reproducible for a given (seed, id, device type).


def _gen(device, seed: int):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def torch_dtype(spec: Spec):
    """Query / output (and new K/V) dtype."""
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[spec.dtype]


def torch_kv_dtype(spec: Spec):
    """Cache storage dtype."""
    import torch
    return torch.float8_e4m3fn if spec.fp8 else torch_dtype(spec)


def kv_content(spec: Spec, kv_id: int, n: int, device="cpu", spikes: "SpikePlan" = None):
    """K and V of n appended tokens, [n, Hkv, D] each, N(0,1) in the cache dtype;
    with a spike plan, the planned tokens of this draw carry their spike."""
    import torch
    g = _gen(device, spec.seed * 1_000_003 + 7919 * kv_id + 17)
    shape = (n, spec.Hkv, spec.D)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if spikes is not None and spikes.by_kv.get(kv_id):
        sp = spikes.by_kv[kv_id]
        t = torch.tensor([x.t for x in sp], dtype=torch.int64, device=device)
        hg = torch.tensor([x.g for x in sp], dtype=torch.int64, device=device)
        kk = np.stack([x.c / np.sqrt(spec.D) * spikes.q_sign(x.row) for x in sp])
        vv = np.stack([SPIKE_V * spikes.v_sign(x.row) for x in sp])
        k[t, hg] = torch.tensor(kk, dtype=torch.float32, device=device)
        v[t, hg] = torch.tensor(vv, dtype=torch.float32, device=device)
    return k.to(torch_dtype(spec)), v.to(torch_dtype(spec))


def q_content(spec: Spec, B: int, device="cpu", spikes: "SpikePlan" = None):
    """Decode queries [B, Hq, D], N(0,1) in the cache dtype; with a spike plan,
    row (b, h) is the plan's sign vector of row id b * Hq + h."""
    import torch
    if spikes is not None:
        return spike_queries(spikes, B * spec.Hq, spec, device).reshape(B, spec.Hq, spec.D)
    g = _gen(device, spec.seed * 1_000_003 + 5)
    q = torch.randn((B, spec.Hq, spec.D), generator=g, device=device, dtype=torch.float32)
    return q.to(torch_dtype(spec))


# ---------------------------------------------------------------------------
# Boundary-dominant contents for the parity tests.
#
# With N(0,1) contents every token carries about 1/L of the softmax weight, so
# losing, repeating or misplacing one token moves the output by about 1/L,
# far below the output tolerance at realistic lengths.  A spike plan gives each
# query row (b, h) a query that is a vector of signs s (+-1) and places, at one
# chosen position j of its sequence and kv head, a key c / sqrt(D) * s (so the
# row's score there is c, against background scores of about N(0, 1)) and a
# value SPIKE_V * s' (another sign vector).  c = ln(n) + 0.5 for a row that
# attends to n keys puts about half of the row's weight on that one token, so
# dropping it, counting it twice or reading a neighbour in its place changes
# the output by a large fraction of SPIKE_V.  The positions are the ones where
# such slips happen: the first and last token, block edges, partition and
# span edges, tile edges, the last tile of a partition, and for several query
# tokens the key just past a query's causal limit.  Only random draws are
# placed here; no attention is computed.

SPIKE_V = 2.0


@dataclass
class Spike:
    t: int        # token offset inside its append draw
    g: int        # kv head
    row: int      # query row id whose sign vector the key takes
    c: float      # that row's score at this key


@dataclass
class SpikePlan:
    seed: int
    D: int
    by_kv: Dict[int, List[Spike]]                 # kv_id -> spikes inside that draw
    rows: Dict[int, Tuple[int, int, int, str]]    # row id -> (seq index or query token, head, position, kind)

    def q_sign(self, row: int) -> np.ndarray:
        return np.random.default_rng([self.seed, row, 1]).choice([-1.0, 1.0], self.D)

    def v_sign(self, row: int) -> np.ndarray:
        return np.random.default_rng([self.seed, row, 2]).choice([-1.0, 1.0], self.D)


def spike_queries(plan: SpikePlan, n_rows: int, spec: Spec, device="cpu"):
    """[n_rows, D] queries: row r is the plan's sign vector of row id r."""
    import torch
    q = np.stack([plan.q_sign(r) for r in range(n_rows)]) if n_rows else np.zeros((0, spec.D))
    return torch.tensor(q, dtype=torch.float32, device=device).to(torch_dtype(spec))


SPIKE_KINDS = ("end", "start", "partition", "partition", "block", "tile", "last_tile",
               "shared", "shared")


def _spike_candidate(kind, n, bs, parts, rng, shared=0):
    """A position in [0, n) of the given kind, or None if the sequence has none.
    `shared`: tokens its family holds in common; a kernel that serves them once
    for the family splits the sequence at the last whole block inside them and
    partitions the rest from there ("shared" edges)."""
    if kind == "end":
        return n - 1
    if kind == "start":
        return 0
    if kind == "shared":
        S = shared // bs * bs
        if S <= 0 or S >= n:
            return None
        P = int(rng.choice(parts))
        k = int(rng.integers(0, (n - 1 - S) // P + 1))        # the split or a later edge
        return S + k * P - int(rng.integers(0, 2))
    if kind in ("partition", "last_tile"):
        P = int(rng.choice(parts))
        if n <= P:
            return None
        k = int(rng.integers(1, (n - 1) // P + 1))          # an edge k*P inside (0, n)
        if kind == "last_tile":
            return k * P - 1 - int(rng.integers(0, min(128, P)))
        return k * P - int(rng.integers(0, 2))
    step = bs if kind == "block" else int(rng.choice((32, 128)))
    if n <= step:
        return None
    k = int(rng.integers(1, (n - 1) // step + 1))
    return k * step - int(rng.integers(0, 2))


def _locate(segs, j):
    for kv_id, pos0, cnt in segs:
        if pos0 <= j < pos0 + cnt:
            return kv_id, j - pos0
    raise ValueError(f"position {j} is not covered by the sequence's appends")


def spike_plan(sc: Scenario, parts: Sequence[int], seed: int = 0,
               seqs: Optional[Sequence[int]] = None,
               query_lens: Optional[Sequence[int]] = None) -> Scenario:
    """The scenario with a spike plan: one spike for every query row of the
    chosen batch indices (all by default), at a boundary position.

    Decode (query_lens None): row (b, h) attends to positions [0, L_b).
    Several query tokens (query_lens[b] = Q_b): query token i of sequence b (a
    global token index t, rows t * Hq + h) attends to [0, L_b - Q_b + i], and
    a further kind puts its spike just past that limit, at L_b - Q_b + i + 1
    (a key the row must not see).  `parts` are the partition / span lengths
    whose edges matter."""
    spec = sc.spec
    rng = np.random.default_rng([sc.spec.seed, seed, 4431])
    lens = [int(x) for x in sc.context_lens]
    pick = range(len(sc.batch)) if seqs is None else seqs
    by_kv: Dict[int, List[Spike]] = {}
    rows: Dict[int, Tuple[int, int, int, str]] = {}
    taken = set()
    qstart = None
    if query_lens is not None:
        qlens = [min(int(q), L) for q, L in zip(query_lens, lens)]
        qstart = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int64)
    for b in pick:
        L = lens[b]
        segs = sc.segments[sc.batch[b]]
        if query_lens is None:
            units = [(b, L, None)]                    # (row base, keys seen, limit)
        else:
            Qb = int(qstart[b + 1] - qstart[b])
            units = [(int(qstart[b]) + i, L - Qb + i + 1, L) for i in range(Qb)]
        for unit, n, limit in units:
            if n <= 0:
                continue
            for h in range(spec.Hq):
                g = h // spec.G
                row = unit * spec.Hq + h
                for _ in range(24):                   # a few tries for a free position
                    kinds = SPIKE_KINDS + (("past_limit",) if limit is not None else ())
                    kind = kinds[int(rng.integers(0, len(kinds)))]
                    if kind == "past_limit":
                        j = n if n < limit else None
                    else:
                        j = _spike_candidate(kind, n, spec.block_size, parts, rng,
                                             sc.shared.get(sc.batch[b], 0))
                    if j is None or not 0 <= j < L:
                        continue
                    kv_id, t = _locate(segs, j)
                    if (kv_id, t, g) in taken:
                        continue
                    taken.add((kv_id, t, g))
                    c = float(np.log(max(n, 2)) + 0.5)
                    by_kv.setdefault(kv_id, []).append(Spike(t, g, row, c))
                    rows[row] = (unit, h, j, kind)
                    break
    return replace(sc, spikes=SpikePlan(int(rng.integers(1 << 31)), spec.D, by_kv, rows))


def poison_value(spec: Spec):
    """Fill for every cache slot no token was written to (NaN; the E4M3 NaN
    code for E4M3 caches): a kernel that reads an unused tail slot into its
    result turns the output into NaN."""
    return float("nan")


def storage_view(t):
    """A CPU tensor as the numpy array of its stored bits (float32 stays
    float32; fp16 / bf16 become uint16 bit patterns, E4M3 uint8 codes)."""
    import torch
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.view(torch.int16).numpy().view(np.uint16)
