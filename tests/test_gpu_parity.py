"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

encode/decode must match the oracle bit for bit (format bytes included); salr_linear
must satisfy ||Y - Y*||_F <= 4e-3 ||Y*||_F and |Y - Y*| <= 1e-2 * S elementwise, S the
sum of |products| feeding each output.  Small and ragged shapes are compared in full;
the full-size workloads are compared on sampled rows and columns the oracle computes
one by one, plus properties that hold at any size.
"""
import functools

import numpy as np
import pytest

import oracle
import salr_synth as synth
from salr_synth import bf16_bits_to_f64
from gpu_util import assert_close, to_bits, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
salr = pytest.importorskip("sparse_rank_linear_b200")


@pytest.fixture(scope="module", autouse=True)
def lib():
    from sparse_rank_linear_b200.build import build
    build()
    assert torch.cuda.is_available()
    return salr.load_library()


@functools.lru_cache(maxsize=None)
def weight(name):
    return synth.weight(synth.WORKLOADS[name])


@functools.lru_cache(maxsize=None)
def encoded(name, sparsity=0.5):
    W = to_dev(weight(name))
    h = salr.encode(W, sparsity)
    torch.cuda.synchronize()
    return h, W


@functools.lru_cache(maxsize=None)
def adapters_dev(name):
    ad = synth.adapters(synth.WORKLOADS[name])
    acat = np.concatenate([a for a, _ in ad], axis=1)  # caller-side layout: stack along rank
    bcat = np.concatenate([b for _, b in ad], axis=0)
    return ad, to_dev(acat), to_dev(bcat)


def sample_idx(n, extra, seed, count):
    rng = np.random.default_rng(seed)
    idx = set(int(v) for v in extra if 0 <= v < n)
    idx |= set(rng.integers(0, n, size=count).tolist())
    return np.array(sorted(idx))


# ---------------------------------------------------------------- codec

@pytest.mark.parametrize("name", ["tiny", "q_proj"])
def test_encode_bytes_and_decode_bitexact_full(name):
    wl = synth.WORKLOADS[name]
    w = weight(name)
    m = oracle.magnitude_mask(w, 0.5)
    wp = oracle.prune(w, m)
    offs, blob = oracle.encode_format(wp, m)
    h, _ = encoded(name)
    gblob, goffs = h.format_tensors()
    assert (goffs.cpu().numpy().view(np.uint32) == offs).all()
    assert gblob.numel() == blob.size and (gblob.cpu().numpy() == blob).all()
    assert (to_bits(h.decode()) == wp).all()
    inf = h.info()
    assert inf["nnz"] == wl.N * (wl.K // 2)
    assert inf["bytes"] == blob.size + 4 * offs.size


@pytest.mark.parametrize("name", ["up_proj", "down_proj", "large"])
def test_encode_decode_full_size_bitexact(name):
    # every row, every block: decode(encode(W)) against the oracle's pruned weight and the
    # whole blob and offset table against the oracle's encoder, in chunks of row tiles
    wl = synth.WORKLOADS[name]
    h, W = encoded(name)
    dec = h.decode()
    assert h.info()["nnz"] == wl.N * (wl.K // 2)
    gblob, goffs = h.format_tensors()
    goffs = goffs.cpu().numpy().view(np.uint32).astype(np.int64)
    assert goffs[-1] * 16 == gblob.numel()
    kb = wl.K // 64
    w_all = weight(name)
    rows_per_chunk = 2048
    for r0 in range(0, wl.N, rows_per_chunk):
        r1 = min(wl.N, r0 + rows_per_chunk)
        w = w_all[r0:r1]
        m = oracle.magnitude_mask(w, 0.5)
        wp = oracle.prune(w, m)
        assert (to_bits(dec[r0:r1]) == wp).all(), f"decode rows {r0}..{r1}"
        o, b = oracle.encode_format(wp, m)
        t0, t1 = r0 // 128, r1 // 128
        lo, hi = goffs[t0 * kb], goffs[t1 * kb]
        assert (goffs[t0 * kb:t1 * kb + 1] - lo == o).all(), f"offsets rows {r0}..{r1}"
        assert (gblob[16 * lo:16 * hi].cpu().numpy() == b).all(), f"blob rows {r0}..{r1}"


def test_encode_handworked_block_and_edge_rows():
    # one block (128 x 64): rows of ties, zeros of both signs, infinities
    rng = np.random.default_rng(2)
    vals = rng.choice(np.array([0.0, -0.0, 0.5, -0.5, 1.0, 2.0, -np.inf, np.inf], np.float32),
                      size=(128, 64))
    vals[0] = 0.25          # all equal: the first 32 are kept
    vals[1] = -0.0
    w = synth.f32_to_bf16_bits(vals)
    m = oracle.magnitude_mask(w, 0.5)
    wp = oracle.prune(w, m)
    h = salr.encode(to_dev(w), 0.5)
    assert (to_bits(h.decode()) == wp).all()
    o, b = oracle.encode_format(wp, m)
    gb, go = h.format_tensors()
    assert (go.cpu().numpy().view(np.uint32) == o).all() and (gb.cpu().numpy() == b).all()
    h.free()


@pytest.mark.parametrize("s", [0.0, 0.3, 0.75])
def test_encode_other_sparsities(s):
    wl = synth.Workload("t", 256, 320, (8,), (4,))
    w = synth.weight(wl)
    s32 = float(np.float32(s))
    m = oracle.magnitude_mask(w, s32)
    wp = oracle.prune(w, m)
    h = salr.encode(to_dev(w), s)
    assert (to_bits(h.decode()) == wp).all()
    assert h.info()["nnz"] == 256 * oracle.keep_count(320, s32)
    h.free()


def test_encode_widest_rows():
    # K = 32768, the largest the format allows: the row's keys need 64 KB of shared memory
    wl = synth.Workload("wide", 256, 32768, (8,), (4,))
    w = synth.weight(wl)
    m = oracle.magnitude_mask(w, 0.5)
    wp = oracle.prune(w, m)
    h = salr.encode(to_dev(w), 0.5)
    assert (to_bits(h.decode()) == wp).all()
    o, b = oracle.encode_format(wp, m)
    gb, go = h.format_tensors()
    assert (go.cpu().numpy().view(np.uint32) == o).all() and (gb.cpu().numpy() == b).all()
    x = synth.activations(wl, 4)
    ad = synth.adapters(wl)
    Y = salr.linear(to_dev(x), h, to_dev(ad[0][0]), to_dev(ad[0][1]))
    assert h.sync_status() == 0
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad), "K=32768")
    h.free()


def test_encode_rejects_nan():
    w = synth.weight(synth.Workload("t", 128, 64, (8,), (1,))).copy()
    w[77, 5] = 0x7FC1
    with pytest.raises(salr.SalrError) as e:
        salr.encode(to_dev(w), 0.5)
    assert e.value.code == 1


def test_double_free_rejected():
    h = salr.encode(to_dev(synth.weight(synth.Workload("t", 128, 64, (8,), (1,)))), 0.5)
    raw = h.handle
    h.free()
    assert salr.load_library().salr_free(raw) == 1


# ---------------------------------------------------------------- linear

def run_linear(name, M, rows=None, cols=None, R_on=True):
    wl = synth.WORKLOADS[name]
    h, _ = encoded(name)
    x = synth.activations(wl, M)
    ad, A, B = adapters_dev(name)
    Y = salr.linear(to_dev(x), h, A if R_on else None, B if R_on else None)
    assert h.sync_status() == 0
    y = to_bits(Y)
    ad_used = ad if R_on else []
    if rows is None:
        w = weight(name)
        wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
        ystar = oracle.linear(x, wp, ad_used)
        s = oracle.abs_bound(x, wp, ad_used)
        return assert_close(y, ystar, s, f"{name} M={M}")
    w = weight(name)[cols]
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    adc = [(a, b[:, cols]) for a, b in ad_used]
    ystar = oracle.linear(x[rows], wp, adc)
    s = oracle.abs_bound(x[rows], wp, adc)
    return assert_close(y[np.ix_(rows, cols)], ystar, s, f"{name} M={M} sampled")


@pytest.mark.parametrize("name,M", [("tiny", 16), ("q_proj", 1), ("q_proj", 16)])
def test_linear_full_compare(name, M):
    run_linear(name, M)


def test_linear_no_adapter_q_proj():
    run_linear("q_proj", 16, R_on=False)


@pytest.mark.parametrize("name,M", [("up_proj", 2048), ("down_proj", 1), ("down_proj", 128),
                                    ("down_proj", 4096), ("large", 16), ("large", 8192)])
def test_linear_full_size_sampled(name, M):
    wl = synth.WORKLOADS[name]
    rows = sample_idx(M, [0, M - 1, 255, 256], 3, 40)
    cols = sample_idx(wl.N, [0, 127, 128, wl.N - 1], 4, 200)
    run_linear(name, M, rows, cols)


@pytest.mark.parametrize("M", [16, 64, 128])
def test_linear_graph_replays_match_oracle(M):
    # salr_linear captured once into a CUDA graph and replayed: every replay must give
    # the oracle's layer (the call's scratch is left zero on the device by each call, so
    # nothing the host decided at capture time goes stale)
    name = "q_proj"
    wl = synth.WORKLOADS[name]
    h, _ = encoded(name)
    ad, A, B = adapters_dev(name)
    x = synth.activations(wl, M)
    X = to_dev(x)
    Y = torch.empty(M, wl.N, dtype=torch.bfloat16, device="cuda")
    salr.linear(X, h, A, B, Y=Y)  # first use: the handle's scratch is allocated here
    torch.cuda.synchronize()
    assert h.sync_status() == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        salr.linear(X, h, A, B, Y=Y)
    w = weight(name)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    ystar = oracle.linear(x, wp, ad)
    s = oracle.abs_bound(x, wp, ad)
    for rep in range(3):
        Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert h.sync_status() == 0
        assert_close(to_bits(Y), ystar, s, f"replay {rep} M={M}")
    # an ordinary call after the replays still finds clean scratch
    assert_close(to_bits(salr.linear(X, h, A, B)), ystar, s, f"after replays M={M}")
    del g


@pytest.mark.parametrize("M", [1, 17, 100, 300])
@pytest.mark.parametrize("R", [0, 8, 72, 128])
def test_linear_ragged_shapes(M, R):
    wl = synth.Workload("ragged", 384, 320, (R,) if R else (), (M,))
    w = synth.weight(wl)
    x = synth.activations(wl, M)
    ad = synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    A = to_dev(ad[0][0]) if R else None
    B = to_dev(ad[0][1]) if R else None
    Y = salr.linear(to_dev(x), h, A, B)
    assert h.sync_status() == 0
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad),
                 f"ragged M={M} R={R}")
    # a second call on the same handle reuses the (self-clearing) split-K workspace
    Y2 = salr.linear(to_dev(x), h, A, B)
    assert_close(to_bits(Y2), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad), "repeat")
    h.free()


@pytest.mark.parametrize("N,K,M", [(5120, 256, 2048), (20480, 128, 200)])
@pytest.mark.parametrize("R", [0, 72, 128])
def test_linear_several_units_per_cta_full_compare(R, N, K, M):
    # more units than the at most 148 persistent CTAs: 40 row tiles x 8 token tiles (the
    # dense-scratch weight path) or 160 row tiles x 1 token tile (the fused decode).  CTAs
    # run units back to back through the same rings, with both TMEM accumulators in use
    # and two adapter chunks per unit (R = 72: the second partial)
    wl = synth.Workload("multi", N, K, (R,) if R else (), (M,))
    w, x = synth.weight(wl), synth.activations(wl, M)
    ad = synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    A = to_dev(ad[0][0]) if R else None
    B = to_dev(ad[0][1]) if R else None
    Y = salr.linear(to_dev(x), h, A, B)
    assert h.sync_status() == 0
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad), f"multi R={R}")
    h.free()


@pytest.mark.parametrize("N,K,M", [(5120, 1024, 2048), (20480, 1024, 200)])
@pytest.mark.parametrize("R", [0, 72])
def test_linear_split_tail_tiles_full_compare(R, N, K, M):
    # 320 tiles (dense-scratch path) or 160 tiles (fused decode) of 16 K blocks on 148
    # SMs: the tiles of the last, partial round are split in four along K, their parts
    # summed in the fp32 workspace, with the adapter on each tile's first part.  A second
    # call, and a call with another token count, reuse the self-clearing workspace.
    wl = synth.Workload("tail", N, K, (R,) if R else (), (M,))
    w, x = synth.weight(wl), synth.activations(wl, M)
    ad = synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    A = to_dev(ad[0][0]) if R else None
    B = to_dev(ad[0][1]) if R else None
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    expect, bound = oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad)
    for call in range(2):
        Y = salr.linear(to_dev(x), h, A, B)
        assert h.sync_status() == 0
        assert_close(to_bits(Y), expect, bound, f"tail R={R} call {call}")
    m2 = M // 2 + 3
    Y = salr.linear(to_dev(x[:m2]), h, A, B)
    assert h.sync_status() == 0
    assert_close(to_bits(Y), expect[:m2], bound[:m2], f"tail R={R} M={m2}")
    h.free()


@pytest.mark.parametrize("N,K,M", [(1280, 512, 384), (9728, 256, 384), (9472, 256, 1024),
                                   (9728, 512, 1100)])
@pytest.mark.parametrize("R", [0, 72])
def test_linear_wide_tiles_full_compare(R, N, K, M, monkeypatch):
    # dense path with 256-row tiles (two MMAs per X tile, two TMEM accumulators per unit):
    # every tile split in 8 along K, whole tiles in one partial round, exactly one round,
    # and 148 whole tiles plus 42 split in two with a ragged last token tile.  The library
    # takes such tiles only from 8 full rounds on; the override reaches them here.
    monkeypatch.setenv("SALR_WIDE_MIN_ROUNDS", "0")
    if salr.plan(N, K, M, R)["tile_rows"] != 256:
        pytest.skip("this GPU's SM count gives 128-row tiles for this shape")
    wl = synth.Workload("wide", N, K, (R,) if R else (), (M,))
    w, x = synth.weight(wl), synth.activations(wl, M)
    ad = synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    A = to_dev(ad[0][0]) if R else None
    B = to_dev(ad[0][1]) if R else None
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    expect, bound = oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad)
    for call in range(2):
        Y = salr.linear(to_dev(x), h, A, B)
        assert h.sync_status() == 0
        assert_close(to_bits(Y), expect, bound, f"wide R={R} call {call}")
    h.free()


@pytest.mark.parametrize("N,K,M,g,wide", [(640, 256, 600, 2, False), (1536, 512, 1100, 4, False),
                                          (1280, 512, 1100, 2, True)])
def test_linear_grouped_tile_order_full_compare(N, K, M, g, wide, monkeypatch):
    # output tiles taken in groups of g row tiles, token tile by token tile (the order the
    # library takes when X outgrows the L2), with a short last group and a ragged last
    # token tile, on 128- and 256-row tiles
    monkeypatch.setenv("SALR_TILE_GROUP_ROWS", str(g))
    if wide:
        monkeypatch.setenv("SALR_WIDE_MIN_ROUNDS", "0")
        if salr.plan(N, K, M, 72)["tile_rows"] != 256:
            pytest.skip("this GPU's SM count gives 128-row tiles for this shape")
    wl = synth.Workload("grouped", N, K, (72,), (M,))
    w, x, ad = synth.weight(wl), synth.activations(wl, M), synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.5)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    Y = salr.linear(to_dev(x), h, to_dev(ad[0][0]), to_dev(ad[0][1]))
    assert h.sync_status() == 0
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad),
                 f"grouped tiles g={g}")
    h.free()


@pytest.mark.parametrize("M", [256, 64])
def test_identity_rows_reproduce_decoded_columns_bitexact(M):
    # X = rows of the identity, no adapter: every output is a single product
    K = 256
    wl = synth.Workload("t", 384, K, (8,), (M,))
    w = synth.weight(wl)
    h = salr.encode(to_dev(w), 0.5)
    x = np.zeros((M, K), np.uint16)
    x[np.arange(M), np.arange(M)] = 0x3F80
    Y = salr.linear(to_dev(x), h)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    y = to_bits(Y)
    expect = wp.T[:M].copy()
    # -0 weights give -0 products; a split-K sum of +0 partials may return +0
    assert ((y == expect) | ((expect == 0x8000) & (y == 0))).all()
    h.free()


def test_sparsity_zero_is_dense_gemm():
    wl = synth.Workload("t", 256, 256, (16,), (16,))
    w, x = synth.weight(wl), synth.activations(wl, 16)
    ad = synth.adapters(wl)
    h = salr.encode(to_dev(w), 0.0)
    Y = salr.linear(to_dev(x), h, to_dev(ad[0][0]), to_dev(ad[0][1]))
    assert_close(to_bits(Y), oracle.linear(x, w, ad), oracle.abs_bound(x, w, ad), "dense")
    h.free()


@pytest.mark.parametrize("s", [0.0, 0.3, 0.75])
@pytest.mark.parametrize("M", [16, 300])
def test_linear_other_sparsities(s, M):
    # the block sizes follow s (17 KB for a dense block, about 5 KB at s = 0.75): both
    # kernels size their compact-block ring slots from the handle's largest block
    wl = synth.Workload("t", 640, 1152, (64, 16), (M,))
    w, x = synth.weight(wl), synth.activations(wl, M)
    ad = synth.adapters(wl)
    acat = np.concatenate([a for a, _ in ad], axis=1)
    bcat = np.concatenate([b for _, b in ad], axis=0)
    s32 = float(np.float32(s))
    h = salr.encode(to_dev(w), s)
    Y = salr.linear(to_dev(x), h, to_dev(acat), to_dev(bcat))
    assert h.sync_status() == 0
    wp = oracle.prune(w, oracle.magnitude_mask(w, s32))
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad),
                 f"s={s} M={M}")
    h.free()


def test_linear_q_proj_sparsity_0p3_full_compare():
    wl = synth.WORKLOADS["q_proj"]
    w, x = weight("q_proj"), synth.activations(wl, 16)
    ad, A, B = adapters_dev("q_proj")
    s32 = float(np.float32(0.3))
    h = salr.encode(to_dev(w), 0.3)
    assert h.info()["nnz"] == wl.N * oracle.keep_count(wl.K, s32)
    Y = salr.linear(to_dev(x), h, A, B)
    assert h.sync_status() == 0
    wp = oracle.prune(w, oracle.magnitude_mask(w, s32))
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad), "q_proj s=0.3")
    h.free()


def test_linear_host_matches_device_path():
    name, M = "q_proj", 16
    h, _ = encoded(name)
    _, A, B = adapters_dev(name)
    x = synth.activations(synth.WORKLOADS[name], M)
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty(M, 4096, dtype=torch.bfloat16).pin_memory()
    salr.linear_host(xh, h, A, B, yh)
    torch.cuda.synchronize()
    yd = salr.linear(to_dev(x), h, A, B)
    w = weight(name)
    wp = oracle.prune(w, oracle.magnitude_mask(w, 0.5))
    ad = synth.adapters(synth.WORKLOADS[name])
    assert_close(to_bits(yh), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad), "host")
    assert_close(to_bits(yd), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad), "device")


def test_linear_rejects_unsupported_rank():
    h, _ = encoded("tiny")
    x = to_dev(synth.activations(synth.WORKLOADS["tiny"], 4))
    A = torch.zeros(256, 12, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(12, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(salr.SalrError) as e:
        salr.linear(x, h, A, B)
    assert e.value.code == 2


# ---------------------------------------------------------------- serialised image

import image_util  # noqa: E402


@pytest.mark.parametrize("name,s", [("tiny", 0.5), ("q_proj", 0.5), ("q_proj", 0.3)])
def test_save_writes_the_documented_image(name, s):
    w = weight(name)
    h = salr.encode(to_dev(w), s)
    img = h.to_bytes()
    assert img == image_util.image(w, s)
    h.free()


def test_load_of_an_oracle_image_is_the_encoded_weight():
    # the image is built by the oracle alone: salr_load must rebuild the handle that
    # salr_encode would give
    name = "q_proj"
    wl = synth.WORKLOADS[name]
    w = weight(name)
    img = image_util.image(w, 0.5)
    h = salr.load(img)
    m = oracle.magnitude_mask(w, 0.5)
    wp = oracle.prune(w, m)
    assert (to_bits(h.decode()) == wp).all()
    offs, blob = oracle.encode_format(wp, m)
    gblob, goffs = h.format_tensors()
    assert (goffs.cpu().numpy().view(np.uint32) == offs).all()
    assert (gblob.cpu().numpy() == blob).all()
    assert h.info() == {"N": wl.N, "K": wl.K, "nnz": wl.N * wl.K // 2,
                        "bytes": blob.size + 4 * offs.size}
    assert h.to_bytes() == img
    x = synth.activations(wl, 16)
    ad, A, B = adapters_dev(name)
    Y = salr.linear(to_dev(x), h, A, B)
    assert h.sync_status() == 0
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad), "loaded")
    h.free()


@pytest.mark.parametrize("M", [16, 300])
def test_save_load_round_trip_serves_the_layer(M):
    wl = synth.Workload("t", 640, 1152, (64, 16), (M,))
    w, x = synth.weight(wl), synth.activations(wl, M)
    ad = synth.adapters(wl)
    acat = np.concatenate([a for a, _ in ad], axis=1)
    bcat = np.concatenate([b for _, b in ad], axis=0)
    h0 = salr.encode(to_dev(w), 0.3)
    img = h0.to_bytes()
    h0.free()
    h = salr.load(img)
    Y = salr.linear(to_dev(x), h, to_dev(acat), to_dev(bcat))
    assert h.sync_status() == 0
    wp = oracle.prune(w, oracle.magnitude_mask(w, float(np.float32(0.3))))
    assert_close(to_bits(Y), oracle.linear(x, wp, ad), oracle.abs_bound(x, wp, ad),
                 f"round trip M={M}")
    h.free()


def test_load_rejects_images_that_fail_the_device_checks():
    # offsets stay valid, so every read of the checks stays inside its block
    w = weight("tiny")
    good = image_util.image(w, 0.5)
    f, offs, blob = image_util.split(good)
    n, k, keep, nnz, s = f[3], f[4], f[5], f[6], f[7]

    def with_blob(b):
        return image_util.pack(n, k, keep, nnz, s, offs, b)

    def rejected(img):
        with pytest.raises(salr.SalrError) as e:
            salr.load(img)
        return e.value.code == salr.binding.SALR_ERR_INVALID

    o = offs.astype(np.int64) * 16
    words = lambda b, blk: b[o[blk]:o[blk] + 1024].view("<u8")  # noqa: E731
    # 1. eight more bits in a bitmap (16 more value bytes): the population no longer
    #    gives the block's size
    b = blob.copy()
    wv = words(b, 0)
    for free in np.flatnonzero(((wv[0] >> np.arange(64, dtype=np.uint64)) & 1) == 0)[:8]:
        wv[0] |= np.uint64(1) << np.uint64(int(free))
    assert rejected(with_blob(b))
    # 2. a bit moved from row 0 to row 1 of a block: same size, wrong row counts
    b = blob.copy()
    wv = words(b, 0)
    bits0 = (wv[0] >> np.arange(64, dtype=np.uint64)) & 1
    bits1 = (wv[1] >> np.arange(64, dtype=np.uint64)) & 1
    c = int(np.flatnonzero((bits0 == 1) & (bits1 == 0))[0])
    wv[0] &= ~(np.uint64(1) << np.uint64(c))
    wv[1] |= np.uint64(1) << np.uint64(c)
    assert rejected(with_blob(b))
    # 3. a kept value that is NaN
    b = blob.copy()
    b[o[3] + 1024:o[3] + 1026] = [0xC1, 0x7F]
    assert rejected(with_blob(b))
    # 4. non-zero padding after the values of a block that has some
    blocks = len(offs) - 1
    pops = [sum(bin(int(x)).count("1") for x in words(blob, i)) for i in range(blocks)]
    i = next(i for i in range(blocks) if (1024 + 2 * pops[i]) % 16)
    b = blob.copy()
    b[o[i + 1] - 1] = 1
    assert rejected(with_blob(b))
    # the untouched image still loads
    salr.load(good).free()
