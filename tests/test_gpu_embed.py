"""Parity of the Q4_K embedding lookup and row gather (through the C ABI) with
the CPU oracle, on a B200: bit-exact f32, every value fl32(w * embed_scale)."""
import numpy as np
import pytest

import oracle
import q4k_synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4k():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gguf_quant_dequant_q4k_b200 as lib
    return lib


def table_problem(rows, hidden, seed):
    w, _ = q4k_synth.q4k_problem(rows, hidden, 1, seed)
    return w


def lookup(q4k, tt, rows, hidden, token, scale):
    out = torch.full((hidden,), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_embed_lookup_f32(tt, rows, hidden, hidden, token, scale, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def assert_same_bits(got, ref, what):
    g = np.asarray(got, np.float32).view(np.uint32)
    r = np.asarray(ref, np.float32).view(np.uint32)
    bad = g != r
    assert not bad.any(), f"{what}: {bad.sum()} values differ"


@pytest.mark.parametrize("rows,hidden", [(256, 256), (300, 1536), (64, 4096), (7, 14336)])
def test_lookup_matches_oracle(q4k, rows, hidden):
    table = table_problem(rows, hidden, 21)
    tt = torch.from_numpy(table).cuda()
    for token in sorted({0, 1, rows // 2, rows - 1}):
        for scale in (1.0, 0.03125, -1.75, float(np.float32(1.0 / np.sqrt(hidden))), 0.0):
            got = lookup(q4k, tt, rows, hidden, token, scale)
            st, ref = oracle.embed_lookup(table, rows, hidden, hidden, token, scale)
            assert st == oracle.EMBED_OK
            assert_same_bits(got, ref, f"{rows}x{hidden} token {token} scale {scale}")


def test_lookup_vocab_table_sampled(q4k):
    """A 128256 x 4096 table (an 8B model's token embedding shape): first, last
    and random tokens, scale 1 and a model-like scale."""
    rows, hidden = 128256, 4096
    table = table_problem(rows, hidden, q4k_synth.SEEDS[(rows, hidden)])
    tt = torch.from_numpy(table).cuda()
    rng = np.random.default_rng(5)
    for token in [0, rows - 1] + rng.integers(0, rows, 6).tolist():
        for scale in (1.0, float(np.float32(64.0 ** 0.5))):
            got = lookup(q4k, tt, rows, hidden, int(token), scale)
            st, ref = oracle.embed_lookup(table, rows, hidden, hidden, int(token), scale)
            assert st == oracle.EMBED_OK
            assert_same_bits(got, ref, f"token {token}")


def test_gather_matches_oracle(q4k):
    rows, hidden = 1000, 2048
    table = table_problem(rows, hidden, 22)
    tt = torch.from_numpy(table).cuda()
    tokens = np.array([0, 999, 5, 5, 512, 1, 998, 0, 777], np.int32)   # duplicates, ends
    out = torch.full((tokens.size, hidden), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_embed_gather_f32(tt, rows, hidden, torch.from_numpy(tokens).cuda(), tokens.size,
                             0.5, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for i, t in enumerate(tokens):
        st, ref = oracle.embed_lookup(table, rows, hidden, hidden, int(t), 0.5)
        assert st == oracle.EMBED_OK
        assert_same_bits(got[i], ref, f"row {i} token {t}")
    assert q4k.q4k_device_fault_flags() == 0


def test_gather_token_out_of_range_raises_flag(q4k):
    """A token outside the table: its row is zeros, the others are exact, and
    the device fault flag says so (then reads back clear)."""
    rows, hidden = 50, 512
    table = table_problem(rows, hidden, 23)
    tt = torch.from_numpy(table).cuda()
    tokens = np.array([3, 50, -1, 49], np.int32)
    out = torch.full((tokens.size, hidden), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_embed_gather_f32(tt, rows, hidden, torch.from_numpy(tokens).cuda(), tokens.size,
                             2.0, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert q4k.q4k_device_fault_flags() == q4k.Q4K_FAULT_TOKEN_RANGE
    assert q4k.q4k_device_fault_flags() == 0
    assert not got[1].any() and not got[2].any()
    for i in (0, 3):
        st, ref = oracle.embed_lookup(table, rows, hidden, hidden, int(tokens[i]), 2.0)
        assert_same_bits(got[i], ref, f"row {i}")


def test_lookup_refusals_launch_nothing(q4k):
    rows, hidden = 16, 256
    table = table_problem(rows, hidden, 24)
    tt = torch.from_numpy(table).cuda()
    out = torch.full((hidden,), 7.0, dtype=torch.float32, device="cuda")
    assert (q4k.q4k_embed_lookup_f32_status(tt, rows, hidden, hidden, rows, 1.0, out)
            == q4k.Q4K_ERR_RANGE)
    assert (q4k.q4k_embed_lookup_f32_status(tt, rows, 512, hidden, 0, 1.0, out)
            == q4k.Q4K_ERR_SHAPE)
    assert (q4k.q4k_embed_lookup_f32_status(tt, rows, hidden, hidden, 0, 1.0, out,
                                            table_bytes=tt.numel() - 144) == q4k.Q4K_ERR_SHAPE)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
