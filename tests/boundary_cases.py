"""Boundary-dominant parity cases, shared by the GPU parity tests
(test_gpu_boundary.py) and the CPU tests that prove each case sensitive
(test_boundary_sensitivity.py).

Every case is a seeded workload whose query rows each carry one spike (see
``workloads.spike_plan``): a key aligned with the row's query at a position
where a kernel could lose, repeat or misplace a token -- the first and last
token, block edges, partition and span edges, tile edges, the last tile of a
partition, and for several query tokens the key just past a query's causal
limit.  The spike holds about half of the row's softmax weight, so a one-token
slip there moves the output far beyond the tolerance ("PagedAttention의 설계"
on the supersilo.blog vLLM summary: one softmax over every valid token, in
logical order).

Contents are drawn on the CPU so that the GPU test and the CPU proof see the
same bytes.
"""
import zlib
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np

import workloads as W

# context lengths spanning several blocks (8/16/32), tiles (32/128), partitions
# (128/512) and one 4096-token partition edge
LENS = (1, 2, 17, 127, 129, 511, 513, 1000, 2049, 4097, 6000, 700)


@dataclass(frozen=True)
class Case:
    name: str
    dtype: str                 # query / output dtype
    G: int
    bs: int
    P: int                     # partition length the kernel runs with
    fp8: bool = False
    D: int = 128
    Hkv: int = 0               # 0: 4 for G <= 2, else 2
    lens: Tuple[int, ...] = LENS
    num_seqs: int = 0          # > 0: uniform lengths ctx_lo..ctx_hi instead of `lens`
    ctx_hi: int = 2000
    spike_every: int = 1       # spike the rows of every n-th sequence
    query_lens: Optional[Tuple[int, ...]] = None   # several query tokens per sequence

    @property
    def hkv(self):
        return self.Hkv or (4 if self.G <= 2 else 2)

    def spec(self) -> W.Spec:
        if self.num_seqs:
            s = W.Spec(self.name, self.dtype, self.G * self.hkv, self.hkv, self.D, self.bs,
                       "independent", self.num_seqs, seed=hash_seed(self.name),
                       ctx_dist="uniform", ctx_lo=1, ctx_hi=self.ctx_hi, partition_size=self.P)
        else:
            s = W.Spec(self.name, self.dtype, self.G * self.hkv, self.hkv, self.D, self.bs,
                       "independent", len(self.lens), seed=hash_seed(self.name),
                       ctx_dist="explicit", ctx_list=self.lens, partition_size=self.P)
        return W.fp8(s) if self.fp8 else s

    def scenario(self) -> W.Scenario:
        sc = W.scenario(self.spec())
        seqs = range(0, len(sc.batch), self.spike_every)
        # the edges of the kernel's partition, of 4096-token spans, and of the
        # 512-token default
        parts = tuple(sorted({self.P, 4096, 512}))
        return W.spike_plan(sc, parts, seed=1, seqs=seqs, query_lens=self.query_lens)


def hash_seed(name: str) -> int:
    return zlib.crc32(name.encode()) % 100_000 + 17


def stream_lens(longest: int, seed: int) -> Tuple[int, ...]:
    """320 context lengths whose grid (320 sequences x 4 kv heads, sized by the
    longest) makes the tcgen05 kernels stream several partitions per CTA, while
    most sequences stay short so the oracle's share of the work stays small:
    every 16th sequence is long (up to `longest`), the rest U[1, 300]."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 301, size=320)
    lens[::16] = rng.integers(longest // 2, longest + 1, size=20)
    lens[0] = longest
    return tuple(int(x) for x in lens)


DECODE = [
    # CUDA-core kernel: f32 / D 64, and G = 1, 2 at 16-bit
    Case("b_f32_g1_d64", "f32", 1, 16, 128, D=64),
    Case("b_f16_g1_p128", "f16", 1, 16, 128),
    Case("b_f16_g1_p512", "f16", 1, 16, 512),
    Case("b_f16_g1_p4096", "f16", 1, 16, 4096),
    Case("b_bf16_g2_p512", "bf16", 2, 16, 512),
    # tcgen05 kernel (G = 4, 8)
    Case("b_bf16_g4_p128", "bf16", 4, 16, 128),
    Case("b_bf16_g4_p512", "bf16", 4, 16, 512),
    Case("b_bf16_g4_p4096", "bf16", 4, 16, 4096),
    Case("b_bf16_g8_p128", "bf16", 8, 16, 128),
    Case("b_bf16_g8_p512", "bf16", 8, 16, 512),
    Case("b_bf16_g8_p4096", "bf16", 8, 16, 4096),
    Case("b_f16_g8_p512", "f16", 8, 16, 512),
    # block sizes 8 and 32
    Case("b_bf16_g8_bs8_p128", "bf16", 8, 8, 128),
    Case("b_f16_g1_bs8_p128", "f16", 1, 8, 128),
    Case("b_bf16_g4_bs32_p512", "bf16", 4, 32, 512),
    Case("b_f16_g1_bs32_p256", "f16", 1, 32, 256),
    # E4M3 caches: CUDA-core (G = 1) and tcgen05 (G = 4, 8)
    Case("b_e4m3_g1_p128", "bf16", 1, 16, 128, fp8=True),
    Case("b_e4m3_g1_p512", "f16", 1, 16, 512, fp8=True),
    Case("b_e4m3_g1_p4096", "bf16", 1, 16, 4096, fp8=True),
    Case("b_e4m3_f32_g1_d64", "f32", 1, 16, 128, fp8=True, D=64),
    Case("b_e4m3_g4_p128", "f16", 4, 16, 128, fp8=True),
    Case("b_e4m3_g4_p512", "f16", 4, 16, 512, fp8=True),
    Case("b_e4m3_g8_p4096", "bf16", 8, 16, 4096, fp8=True),
    Case("b_e4m3_g8_bs8_p512", "bf16", 8, 8, 512, fp8=True),
    Case("b_e4m3_g4_bs32_p128", "bf16", 4, 32, 128, fp8=True),
    # several partitions streamed by one CTA with one softmax: the grid has
    # >= 8 CTAs per SM (320 sequences x 4 kv heads), so spans of 8 x 128 and
    # 8 x 512 tokens
    Case("b_stream_bf16_g8_p128", "bf16", 8, 16, 128, Hkv=4, lens=stream_lens(2000, 1),
         spike_every=4),
    Case("b_stream_bf16_g4_p512", "bf16", 4, 16, 512, Hkv=4, lens=stream_lens(4096, 2),
         spike_every=4),
    Case("b_stream_e4m3_g8_p128", "bf16", 8, 16, 128, fp8=True, Hkv=4,
         lens=stream_lens(2000, 3), spike_every=4),
]

# several query tokens per sequence (verify: few; prefill: a whole chunk)
MQ_LENS = (5, 40, 300, 513, 1100, 2000, 129, 700)
MULTI = [
    Case("m_verify_g8_p128", "bf16", 8, 16, 128, lens=MQ_LENS, query_lens=(1, 2, 2, 1, 2, 2, 1, 2)),
    Case("m_verify_g4_p512", "f16", 4, 16, 512, lens=MQ_LENS, query_lens=(1, 4, 2, 3, 4, 1, 4, 3)),
    Case("m_verify_g8_q8_p512", "bf16", 8, 16, 512, lens=MQ_LENS, query_lens=(1, 8, 5, 8, 3, 8, 2, 7)),
    Case("m_verify_g1_p128", "f16", 1, 16, 128, lens=MQ_LENS, query_lens=(1, 4, 8, 3, 8, 5, 2, 6)),
    # 32 (query token, head) columns: one CTA of the N = 32 kernel per sequence
    Case("m_verify_g8_q4_p256", "bf16", 8, 16, 256, lens=MQ_LENS, query_lens=(4, 3, 4, 1, 4, 2, 4, 3)),
    Case("m_verify_g4_q8_bs8_p128", "f16", 4, 8, 128, lens=MQ_LENS,
         query_lens=(8, 5, 8, 1, 7, 8, 3, 8)),
    Case("m_prefill_g1_p256", "bf16", 1, 16, 256, lens=(200, 700, 1500, 90),
         query_lens=(200, 300, 260, 90)),
    Case("m_prefill_g4_bs8_p128", "bf16", 4, 8, 128, lens=(200, 700, 1500, 90),
         query_lens=(130, 300, 200, 90)),
    Case("m_prefill_g8_bs32_p256", "f16", 8, 32, 256, lens=(200, 700, 1500, 90),
         query_lens=(64, 200, 100, 90)),
]


def mq_offsets(case: Case, lens):
    qlens = np.minimum(np.asarray(case.query_lens, dtype=np.int64), np.asarray(lens, np.int64))
    return np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)


def mq_queries(case: Case, sc: W.Scenario, device="cpu"):
    """[total_q, Hq, D] queries of a multi-query case: row (t, h) is the spike
    plan's sign vector of row id t * Hq + h."""
    spec = sc.spec
    qs = mq_offsets(case, sc.context_lens)
    T = int(qs[-1])
    return W.spike_queries(sc.spikes, T * spec.Hq, spec, device).reshape(T, spec.Hq, spec.D), qs


@dataclass(frozen=True)
class GroupCase:
    """A batch of families sharing leading blocks (pa_decode_grouped): parallel
    samples of a few prompts, or requests forked from one prefix."""
    name: str
    kind: str                  # "parallel_sampling" | "shared_prefix"
    dtype: str
    G: int
    bs: int
    P: int
    Hkv: int = 2
    prompts: int = 3           # parallel sampling
    samples: int = 6
    prompt_lo: int = 200
    prompt_hi: int = 1100
    div_hi: int = 300
    requests: int = 6          # shared prefix
    prefix: int = 1024
    suffix_hi: int = 1800
    spike_every: int = 1
    fp8: bool = False          # E4M3 cache (pa_decode_grouped_fp8)

    def spec(self) -> W.Spec:
        common = dict(name=self.name, dtype=self.dtype, Hq=self.G * self.Hkv, Hkv=self.Hkv, D=128,
                      block_size=self.bs, seed=hash_seed(self.name), partition_size=self.P)
        if self.kind == "parallel_sampling":
            s = W.Spec(kind=self.kind, num_seqs=self.prompts * self.samples,
                       num_prompts=self.prompts, samples_per_prompt=self.samples,
                       prompt_lo=self.prompt_lo, prompt_hi=self.prompt_hi, div_lo=1,
                       div_hi=self.div_hi, **common)
        else:
            s = W.Spec(kind=self.kind, num_seqs=self.requests, prefix_len=self.prefix,
                       suffix_lo=1, suffix_hi=self.suffix_hi, **common)
        return W.fp8(s) if self.fp8 else s

    def scenario(self) -> W.Scenario:
        sc = W.scenario(self.spec())
        parts = tuple(sorted({self.P, 4096, 512}))
        return W.spike_plan(sc, parts, seed=1, seqs=range(0, len(sc.batch), self.spike_every))


GROUPED = [
    # parallel samples of a prompt (the llama13b_ps shape, scaled down): G = 1, 2
    GroupCase("g_ps_g1_p128", "parallel_sampling", "bf16", 1, 16, 128, Hkv=4),
    GroupCase("g_ps_g1_p512", "parallel_sampling", "f16", 1, 16, 512, Hkv=4),
    GroupCase("g_ps_g1_bs8_p128", "parallel_sampling", "bf16", 1, 8, 128, Hkv=4),
    GroupCase("g_ps_g1_bs32_p256", "parallel_sampling", "f16", 1, 32, 256, Hkv=4),
    GroupCase("g_ps_g1_20samples", "parallel_sampling", "bf16", 1, 16, 256, Hkv=2, prompts=2,
              samples=20),
    GroupCase("g_ps_g2_p256", "parallel_sampling", "bf16", 2, 16, 256, Hkv=2),
    GroupCase("g_ps_g8_p128", "parallel_sampling", "bf16", 8, 16, 128, Hkv=2),
    # families of at most 8 / G members: span CTAs with 8 of the 16 columns in use
    GroupCase("g_ps_g2_4samples", "parallel_sampling", "f16", 2, 16, 256, Hkv=2, samples=4),
    GroupCase("g_lp_g4_2requests", "shared_prefix", "bf16", 4, 16, 512, requests=2),
    # requests forked from one prefix (the long_prefix shape, scaled down): G = 4, 8
    GroupCase("g_lp_g4_p512", "shared_prefix", "bf16", 4, 16, 512),
    GroupCase("g_lp_g4_p128", "shared_prefix", "bf16", 4, 16, 128),
    GroupCase("g_lp_g4_bs8_p512", "shared_prefix", "bf16", 4, 8, 512),
    GroupCase("g_lp_g4_bs32_p128", "shared_prefix", "f16", 4, 32, 128),
    GroupCase("g_lp_g8_p256", "shared_prefix", "f16", 8, 16, 256),
    GroupCase("g_lp_g1_p512", "shared_prefix", "bf16", 1, 16, 512, Hkv=4),
    # enough requests that both the span and the rest stream several partitions
    # per CTA (>= 8 CTAs per SM)
    GroupCase("g_lp_g4_stream", "shared_prefix", "bf16", 4, 16, 128, Hkv=4, requests=300,
              prefix=1024, suffix_hi=1800, spike_every=10),
    # E4M3 caches: the spans on the tcgen05 E4M3 kernel with (member, head)
    # columns; the rest on the E4M3 tensor-core kernel (G = 4, 8) or the
    # CUDA-core kernel (G = 1, 2), each past its shift
    GroupCase("g_e4m3_ps_g1_p128", "parallel_sampling", "bf16", 1, 16, 128, Hkv=4, fp8=True),
    GroupCase("g_e4m3_ps_g2_p256", "parallel_sampling", "f16", 2, 16, 256, Hkv=2, fp8=True),
    GroupCase("g_e4m3_ps_g1_20samples", "parallel_sampling", "f16", 1, 16, 512, Hkv=2,
              prompts=2, samples=20, fp8=True),
    GroupCase("g_e4m3_lp_g4_p512", "shared_prefix", "bf16", 4, 16, 512, fp8=True),
    GroupCase("g_e4m3_ps_g2_4samples", "parallel_sampling", "bf16", 2, 16, 128, Hkv=2, samples=4,
              fp8=True),
    GroupCase("g_e4m3_lp_g4_2requests", "shared_prefix", "f16", 4, 16, 256, requests=2, fp8=True),
    GroupCase("g_e4m3_lp_g4_bs32_p128", "shared_prefix", "f16", 4, 32, 128, fp8=True),
    GroupCase("g_e4m3_lp_g8_bs8_p256", "shared_prefix", "bf16", 8, 8, 256, fp8=True),
    GroupCase("g_e4m3_lp_g4_stream", "shared_prefix", "bf16", 4, 16, 128, Hkv=4, requests=300,
              prefix=1024, suffix_hi=1800, spike_every=10, fp8=True),
]
