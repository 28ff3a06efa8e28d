"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bit-exact: expert ids, counts, offsets, sorted_pairs, pair_pos.
Floating point: max|gpu - oracle| / max|oracle| <= 1e-2 per bf16 output tensor
(fp32 accumulation, bf16 storage), routing weights within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import mixture_experts_lora_b200 as ml
import oracle.moe_lora_oracle as O
from moe_inputs import CONFIGS, LayerConfig, small_config, generate

from gpu_common import (TOL, TOL_W, check_full_parity, check_sampled_parity, ensure_built,
                        inputs_on, rel_err, run_layer, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


# ------------------------------------------------------------------ routing
@pytest.mark.parametrize("T,E,k", [(300, 64, 8), (37, 8, 8), (64, 1024, 32), (5, 128, 1), (129, 33, 3)])
def test_route_topk_bitexact_with_ties(T, E, k):
    g = torch.Generator().manual_seed(T * 1000 + E)
    logits = (torch.randn(T, E, generator=g) * 2).round() / 2        # many exact ties
    logits[0] = 0.0                                                  # a fully tied row
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    ml.moe_route_topk(logits.cuda(), k, ids, w)
    torch.cuda.synchronize()
    rid, rw = O.route_topk(logits.numpy(), k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert rel_err(to_np(w), rw) <= TOL_W
    assert np.array_equal(ids[0].cpu().numpy(), np.arange(k))


# ------------------------------------------------------------------ permute
@pytest.mark.parametrize("T,k,E,hot", [(1500, 3, 7, True), (4096, 8, 128, False), (33, 1, 1024, False),
                                        (2000, 4, 16, True)])
def test_permute_bitexact(T, k, E, hot):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    if hot:
        ids[:, 0] = 1
        ids[:, 1:][ids[:, 1:] == 1] = 0
    ids_d = torch.from_numpy(ids).cuda()
    P = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(P, dtype=torch.int32, device="cuda")
    pos = torch.empty(P, dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    ml.moe_permute(ids_d, E, counts, offsets, sp, pos, ws)
    assert ml.moe_get_device_error() == ml.MOE_OK
    rc, ro, rsp, rpos = O.permute(ids, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(sp.cpu().numpy(), rsp)
    assert np.array_equal(pos.cpu().numpy(), rpos)


@pytest.mark.parametrize("T,E,k,hot", [(4096, 128, 8, False), (300, 64, 3, False),
                                       (64, 1024, 32, False), (1000, 16, 1, False),
                                       (129, 33, 5, False), (1, 8, 2, False), (0, 8, 2, False),
                                       (40000, 128, 8, False), (20000, 512, 4, False),
                                       (16384, 128, 8, True), (3001, 96, 3, True)])
def test_route_permute_fused_bitexact(T, E, k, hot):
    # routing and the counting sort in one call: the same ids, weights and permutation
    # as the oracle (and as moe_route_topk followed by moe_permute), ties included.
    # The two large cases need more chunks than resident CTAs (a CTA scatters several)
    # and more tokens than routing warps (a warp routes several, E > 256 reusing its
    # shared logits row).  The hot cases bias the logits towards the low experts, so
    # nearly every token picks the same few (the counts of a token group pile up on
    # one expert; tpc = 170 at k = 3 puts group boundaries inside chunks).
    g = torch.Generator().manual_seed(T * 7 + E + k)
    logits = (torch.randn(T, E, generator=g) * 2).round() / 2
    if hot:
        logits = logits + 8.0 / (1.0 + torch.arange(E, dtype=torch.float32))
    if T > 0:
        logits[0] = 0.0
    P = T * k
    d = lambda *shape, dt=torch.int32: torch.full(shape, -1, dtype=dt, device="cuda")
    ids, w = d(T, k), d(T, k, dt=torch.float32)
    counts, offsets, sp, pos = d(E), d(E + 1), d(P), d(P)
    ws = torch.empty(ml.moe_workspace_bytes(ml.make_dims(max(T, 1), 64, 64, E, k, 16, 1.0)),
                     dtype=torch.uint8, device="cuda")
    ml.moe_route_permute(logits.cuda(), k, ids, w, counts, offsets, sp, pos, ws)
    assert ml.moe_get_device_error() == ml.MOE_OK
    rid, rw = O.route_topk(logits.numpy(), k) if T > 0 else (np.zeros((0, k), np.int64), np.zeros((0, k)))
    rc, ro, rsp, rpos = O.permute(rid, E)
    assert np.array_equal(ids.cpu().numpy(), rid)
    if T > 0:
        assert rel_err(to_np(w), rw) <= TOL_W
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(sp.cpu().numpy(), rsp)
    assert np.array_equal(pos.cpu().numpy(), rpos)
    # the separate calls give the same bits
    ids2, w2 = d(T, k), d(T, k, dt=torch.float32)
    c2, o2, sp2, pos2 = d(E), d(E + 1), d(P), d(P)
    if T > 0:
        ml.moe_route_topk(logits.cuda(), k, ids2, w2)
    ml.moe_permute(ids2, E, c2, o2, sp2, pos2, ws)
    torch.cuda.synchronize()
    for a, b in ((ids, ids2), (counts, c2), (offsets, o2), (sp, sp2), (pos, pos2)):
        assert torch.equal(a, b)
    if T > 0:
        assert torch.equal(w, w2)


def test_permute_reports_bad_expert_id_without_faulting():
    ids = torch.tensor([[0, 1], [2, 7]], dtype=torch.int32, device="cuda")   # 7 >= E
    E = 4
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    pos = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    ml.moe_permute(ids, E, counts, offsets, sp, pos, ws)
    assert ml.moe_get_device_error() == ml.MOE_ERR_DEVICE_INDEX
    assert ml.moe_get_device_error() == ml.MOE_OK        # cleared after reading
    assert counts.cpu().tolist() == [1, 1, 1, 0]


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("weighted", [True, False])
def test_unpermute_combine(weighted):
    T, k, m = 333, 4, 200
    g = torch.Generator().manual_seed(7)
    ys = torch.randn(T * k, m, generator=g).to(torch.bfloat16)
    w = torch.rand(T, k, generator=g)
    pos = torch.randperm(T * k, generator=g).to(torch.int32)
    y = torch.empty(T, m, dtype=torch.bfloat16, device="cuda")
    ml.moe_unpermute_combine(ys.cuda(), w.cuda() if weighted else None, pos.cuda(), T, k, m, y)
    torch.cuda.synchronize()
    ref = O.unpermute_combine(ys.double().numpy(), w.double().numpy() if weighted else None,
                              pos.numpy().astype(np.int64), k)
    # one bf16 rounding of an fp32 sum: within one bf16 ulp of the value
    assert np.all(np.abs(to_np(y) - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)


# ------------------------------------------------------------------ whole layer, tiny + edges
def _layer_case(cfg, mutate=None, seed=0):
    inp, cpu = inputs_on(cfg, seed=seed)
    if mutate is not None:
        mutate(cpu)
        inp = {k: v.cuda().contiguous() for k, v in cpu.items()}
    buf = run_layer(inp, cfg)
    return check_full_parity(buf, cpu, cfg), buf


def test_tiny_config_full_parity():
    errs, _ = _layer_case(CONFIGS["tiny"])
    print("tiny parity", errs)


EDGE = {
    "one_token": small_config(T=1, m=128, n=64, E=8, k=2, r=8, alpha=16),
    "ragged_odd_dims_r16": small_config(T=100, m=144, n=80, E=6, k=2, r=16, alpha=16),
    "partial_gate_tile": small_config(T=150, m=64, n=208, E=4, k=2, r=16, alpha=32),
    "rank32": small_config(T=200, m=128, n=96, E=8, k=2, r=32, alpha=32),
    "rank24_padded": small_config(T=90, m=96, n=48, E=5, k=3, r=24, alpha=48),
    "k_equals_E": small_config(T=70, m=64, n=32, E=8, k=8, r=8, alpha=8),
    "long_K": small_config(T=130, m=1024, n=320, E=4, k=2, r=16, alpha=16),
    # wide ranks: the rank the pages benchmark at (64), the widest supported (128),
    # and ranks padded up to them (48 -> 64, 96 -> 128)
    "rank64": small_config(T=200, m=128, n=96, E=8, k=2, r=64, alpha=64),
    "rank48_padded": small_config(T=90, m=192, n=64, E=5, k=3, r=48, alpha=48),
    "rank128": small_config(T=150, m=256, n=128, E=4, k=2, r=128, alpha=128),
    "rank96_padded_odd_dims": small_config(T=110, m=144, n=80, E=6, k=2, r=96, alpha=96),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_case_full_parity(name):
    errs, _ = _layer_case(EDGE[name])
    print(name, errs)


def test_hot_expert_and_empty_experts():
    cfg = small_config(T=300, m=128, n=64, E=8, k=2, r=8, alpha=16)

    def mutate(cpu):
        cpu["logits"][:, 3] += 20.0          # every token picks expert 3 first
        cpu["logits"][:, 5:] -= 20.0         # experts 5..7 get nothing
    errs, buf = _layer_case(cfg, mutate)
    counts = buf.counts.cpu().numpy()
    assert counts[3] == 300 and counts[5:].sum() == 0


def test_every_tile_size_class():
    # Expert row counts that give every kind of 128-row tile: exact multiples of 128
    # (no short tile), a short tile in each of the four size classes the row kernels
    # order their tiles by (rows >= 96, 64-95, 32-63, < 32), and an empty expert.  n = 96
    # also leaves the SwiGLU kernels a partial 64-column stage.
    counts = [128, 256, 100, 70, 40, 10, 0, 230]
    cfg = small_config(T=sum(counts), m=64, n=96, E=len(counts), k=1, r=16, alpha=16)
    owner = np.repeat(np.arange(len(counts)), counts)
    owner = owner[np.random.default_rng(3).permutation(len(owner))]

    def mutate(cpu):
        cpu["logits"][torch.arange(cfg.T), torch.from_numpy(owner)] += 30.0
    errs, buf = _layer_case(cfg, mutate)
    assert buf.counts.cpu().tolist() == counts
    print(errs)


def test_tied_logits_route_to_lowest_indices():
    cfg = small_config(T=64, m=64, n=32, E=6, k=2, r=8, alpha=16)

    def mutate(cpu):
        cpu["logits"][:] = 0.0
    errs, buf = _layer_case(cfg, mutate)
    assert np.array_equal(buf.ids.cpu().numpy(), np.tile([0, 1], (64, 1)))


def test_deterministic_bitwise():
    cfg = CONFIGS["tiny"]
    inp, cpu = inputs_on(cfg)
    a = run_layer(inp, cfg)
    snap = {k: getattr(a, k).clone() for k in ("Y", "dX", "dA_gu", "dB_gu", "dA_d", "dB_d", "save_GU")}
    b = run_layer(inp, cfg, buf=a)
    for k, v in snap.items():
        assert torch.equal(v.view(torch.int16) if v.dtype == torch.bfloat16 else v,
                           getattr(b, k).view(torch.int16) if v.dtype == torch.bfloat16 else getattr(b, k)), k


def test_empty_input():
    cfg = small_config(T=0, m=64, n=32, E=4, k=2, r=8, alpha=16)
    inp, cpu = inputs_on(cfg)
    buf = ml.alloc_buffers(0, 64, 32, 4, 2, 8, 2.0)
    buf.dA_gu.fill_(1.0)
    ml.layer_step(inp, 2, 2.0, buf)
    assert ml.moe_get_device_error() == ml.MOE_OK
    assert buf.offsets.cpu().tolist() == [0] * 5
    assert not torch.any(buf.dA_gu != 0)


# ------------------------------------------------------------------ full sizes (sampled)
@pytest.mark.parametrize("name", ["qwen3_30b_a3b", "gpt_oss_20b", "qwen3_skewed", "deepseek_v3_e16"])
def test_full_size_sampled_parity(name):
    cfg = CONFIGS[name]
    inp, cpu = inputs_on(cfg)
    buf = run_layer(inp, cfg)
    errs = check_sampled_parity(buf, cpu, cfg)
    print(name, errs)


# Full-size parity in full: every output and saved intermediate of the whole layer,
# element by element, against the oracle run over the whole workload (the oracle
# takes seconds to tens of seconds at these sizes on the host's cores).
@pytest.mark.parametrize("name", ["qwen3_30b_a3b", "qwen3_skewed", "gpt_oss_20b"])
def test_full_size_full_parity(name):
    cfg = CONFIGS[name]
    inp, cpu = inputs_on(cfg)
    buf = run_layer(inp, cfg)
    errs = check_full_parity(buf, cpu, cfg)
    print(name, errs)


def test_skewed_experts_across_two_2048_row_chunks():
    # 1024 rows per expert on average: the adapter-gradient chunk grows to 2048 rows,
    # and the busiest experts (3200-4100 rows under this skew) take two chunks whose
    # partials the last arriving unit sums
    cfg = LayerConfig("skewed_e32", T=4096, m=2048, n=768, E=32, k=8, r=16, alpha=16,
                      zipf_s=1.0, bias_scale=2.0)
    inp, cpu = inputs_on(cfg)
    buf = run_layer(inp, cfg)
    assert int(buf.counts.max()) > 2048
    errs = check_sampled_parity(buf, cpu, cfg, n_tokens=16, n_experts=3)
    print(errs)


def test_expert_spanning_several_chunks():
    # 1500 rows on one expert: several token chunks in the grouped GEMMs and two
    # row chunks in the adapter-gradient reduction
    cfg = small_config(T=1500, m=64, n=48, E=4, k=1, r=16, alpha=16)

    def mutate(cpu):
        cpu["logits"][:, 0] += 30.0
    errs, buf = _layer_case(cfg, mutate)
    assert buf.counts.cpu().tolist()[0] == 1500


@pytest.mark.parametrize("r", [16, 32, 64])
def test_multi_chunk_experts_at_every_rank_width(r):
    # Experts of more than 256 rows are cut into several balanced token chunks of the
    # grouped GEMMs: 257 rows (the smallest cut), 300, 513 (three chunks), 600, next to
    # an expert of one chunk and an empty one.  Rank 16 keeps the GEMMs' LoRA block in
    # its side buffer; ranks 32 and 64 take a ring stage per tile.
    counts = [600, 257, 513, 100, 0, 300]
    cfg = small_config(T=sum(counts), m=128, n=64, E=len(counts), k=1, r=r, alpha=r)
    owner = np.repeat(np.arange(len(counts)), counts)
    owner = owner[np.random.default_rng(5).permutation(len(owner))]

    def mutate(cpu):
        cpu["logits"][torch.arange(cfg.T), torch.from_numpy(owner)] += 30.0
    errs, buf = _layer_case(cfg, mutate)
    assert buf.counts.cpu().tolist() == counts
    print(r, errs)


def test_graph_replay_matches_eager_bitwise():
    # bench.py times CUDA-graph replays of the step (every kernel launched with
    # programmatic dependent launch): a replay must give the eager results bit for bit
    cfg = small_config(T=640, m=256, n=128, E=8, k=2, r=16, alpha=16)
    inp, _ = inputs_on(cfg, seed=11)
    eager = run_layer(inp, cfg)
    keys = ("Y", "dX", "dA_gu", "dB_gu", "dA_d", "dB_d", "save_GU", "save_Xs", "save_H", "Y_sorted")
    snap = {k: getattr(eager, k).clone() for k in keys}
    buf = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r, cfg.scale)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ml.layer_step(inp, cfg.k, cfg.scale, buf)       # warm-up outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            ml.layer_step(inp, cfg.k, cfg.scale, buf)
        for name in keys:
            getattr(buf, name).zero_()
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    assert ml.moe_get_device_error() == ml.MOE_OK
    for k, v in snap.items():
        a = v.view(torch.int16) if v.dtype == torch.bfloat16 else v
        b = getattr(buf, k)
        b = b.view(torch.int16) if b.dtype == torch.bfloat16 else b
        assert torch.equal(a, b), k
    del g


def test_check_permutation_accepts_valid_and_flags_broken():
    T, k, E = 700, 4, 16
    g = torch.Generator().manual_seed(5)
    ids, _ = O.route_topk(torch.randn(T, E, generator=g).numpy(), k)
    d_ids = torch.from_numpy(ids.astype(np.int32)).cuda()
    P = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(P, dtype=torch.int32, device="cuda")
    pos = torch.empty(P, dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    ml.moe_permute(d_ids, E, counts, offsets, sp, pos, ws)
    ml.moe_check_permutation(d_ids, E, counts, offsets, sp, pos)
    assert ml.moe_get_device_error() == ml.MOE_OK

    def broken(mutate):
        c, o, s_, p_ = counts.clone(), offsets.clone(), sp.clone(), pos.clone()
        mutate(c, o, s_, p_)
        ml.moe_check_permutation(d_ids, E, c, o, s_, p_)
        return ml.moe_get_device_error()

    off = offsets.cpu().numpy()
    e = int(np.argmax(np.diff(off)))                       # an expert with at least 2 rows
    q0 = int(off[e])

    def swap_in_segment(c, o, s_, p_):                     # order inside a segment
        a, b = s_[q0].item(), s_[q0 + 1].item()
        s_[q0], s_[q0 + 1] = b, a
        p_[a], p_[b] = q0 + 1, q0

    def bad_offset(c, o, s_, p_):                          # counts disagree with offsets
        o[e + 1] += 1

    def bad_inverse(c, o, s_, p_):                         # pair_pos not the inverse
        p_[0] = (p_[0] + 1) % P

    def out_of_range(c, o, s_, p_):                        # a pair index outside [0, P)
        s_[5] = P + 3

    for mutate in (swap_in_segment, bad_offset, bad_inverse, out_of_range):
        assert broken(mutate) == ml.MOE_ERR_DEVICE_CHECK, mutate.__name__


def test_layer_with_debug_checks(monkeypatch):
    monkeypatch.setenv("MOE_CHECK", "1")
    cfg = CONFIGS["tiny"]
    inp, cpu = inputs_on(cfg)
    buf = run_layer(inp, cfg)                              # every call checked on the device
    check_full_parity(buf, cpu, cfg)
