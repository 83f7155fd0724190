"""The kernel planners' role sets cover the work exactly once (host only).

Read back from the plan's describe() report on every workload (compile-only
plans, no GPU):
  * forward: for each hidden irrep, the roles' channel blocks times their
    path groups cover (channels x paths of the irrep) once, and every role
    sits in one slice;
  * backward: for each hidden irrep with paths, its roles share one phase
    count nph and cover every (32-channel block, edge phase) pair once, all
    in one slice; a slice has no more roles than consumer warps.
The same on irreps sets unlike the workloads, and the one refusal the
planner has (a hidden irrep too wide for shared memory).  And, read from the
generated source, every row copy into shared memory stays inside its global
row and its staging slot, with bulk (TMA) copies on 16-byte boundaries, and
the shared-memory regions are ordered, disjoint, aligned and within the
planned size.
"""
import re
from collections import Counter

import pytest

import oracle as O
from equivariant_mlip_clebsch_b200 import cgtp as C
from equivariant_mlip_clebsch_b200 import workloads as WL

NAMES = ["tiny", "lmax2", "lmax2_wide", "lmax3", "lmax6", "case4", "case5", "case6"]
# irreps sets unlike the workloads: multiplicities 1, 3, 17, 33 and 96 (partial
# warps and blocks), one irrep without any path, missing outputs, odd parities
ODD = [
    ("3x2o", "1x0e+1x1o", "3x1e+3x2o+3x2e+3x3e"),
    ("1x0e", "1x0e+1x1o+1x2e", "1x1o+1x2e"),
    ("96x1e", "1x0e+1x1o", "96x0o+96x1o"),
    ("128x0e+17x1e+1x2e", "1x0e+1x1o+1x2e", "17x0o+129x0e+35x1e+18x2o+147x2e+1x3o+18x3e+1x4e"),
    ("33x0e", "1x0e+1x1o+1x2e+1x3o+1x4e", "33x0e+33x1o+33x3o+33x4e"),
    ("16x0e+16x1o+8x2e", "1x0e+1x1o", "32x0e+16x1e"),  # 8x2e feeds no output
]


@pytest.fixture
def compile_only(monkeypatch):
    monkeypatch.setenv("CGTP_JIT_COMPILE_ONLY", "1")


def _parse(text, kind):
    head = re.search(rf"^{kind}: roles=(\d+) slices=(\d+) warps=(\d+)\+2", text, re.M)
    nroles, nslices, nw = (int(v) for v in head.groups())
    block = text[head.end():]
    slices = []
    for line in block.splitlines():
        m = re.match(r"\s+slice (\d+):((?: \d+)*)\s*$", line)
        if m:
            slices.append([int(v) for v in m.group(2).split()])
        elif slices and not line.startswith("  slice"):
            break
    return nroles, nw, slices[:nslices]


@pytest.mark.parametrize("irreps", [WL.CONFIGS[n] for n in NAMES] + [
    dict(irreps_in=a, irreps_edge=b, irreps_out=c) for a, b, c in ODD], ids=NAMES + [f"odd{k}" for k in range(len(ODD))])
def test_role_coverage(irreps, compile_only):
    c = irreps
    name = c["irreps_in"]
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    text = plan.describe()
    muls = [m for m, _, _ in P.irreps_in]
    npaths = Counter()
    irrep_of_l1 = {}
    for a, (m, l, p) in enumerate(P.irreps_in):
        irrep_of_l1[a] = l
    # path table rows: l1, l2, l3, mul, x_off, k0, o_off, c_off; the hidden
    # irrep of a path is the one whose x block starts at x_off
    x_starts, off = {}, 0
    for a, (m, l, p) in enumerate(P.irreps_in):
        x_starts[off] = a
        off += m * (2 * l + 1)
    for row in P.table:
        npaths[x_starts[int(row[4])]] += 1

    # forward
    nroles, nw, slices = _parse(text, "forward")
    froles = [tuple(int(v) for v in m) for m in
              re.findall(r"frole \d+: irrep (\d+) u0=(\d+) R=(\d+) paths=(\d+)", text)]
    assert len(froles) == nroles
    assert sorted(r for s in slices for r in s) == list(range(nroles))
    assert all(len(s) <= nw for s in slices)
    covered = Counter()
    for a, u0, R, np_ in froles:
        covered[a] += min(32 * R, muls[a] - u0) * np_
    for a in npaths:
        assert covered[a] == muls[a] * npaths[a], (name, a)

    # backward
    nroles, nw, slices = _parse(text, "backward")
    broles = [tuple(int(v) for v in m) for m in
              re.findall(r"brole \d+: irrep (\d+) u0=(\d+) R=(\d+) ph=(\d+)/(\d+)", text)]
    assert len(broles) == nroles
    assert sorted(r for s in slices for r in s) == list(range(nroles))
    assert all(len(s) <= nw for s in slices)
    slice_of = {r: k for k, s in enumerate(slices) for r in s}
    for a in npaths:
        mine = [(i, r) for i, r in enumerate(broles) if r[0] == a]
        assert mine, (name, a)
        assert len({slice_of[i] for i, _ in mine}) == 1  # one slice per irrep
        nph = {r[4] for _, r in mine}
        assert len(nph) == 1
        nph = nph.pop()
        pairs = Counter()
        for _, (_, u0, R, ph, _) in mine:
            for k in range(R):
                if u0 + 32 * k < muls[a]:
                    pairs[(u0 + 32 * k, ph)] += 1
        blocks = range(0, muls[a], 32)
        assert pairs == Counter({(b, ph): 1 for b in blocks for ph in range(nph)}), (name, a)


def test_backward_capacity_refusal(compile_only):
    """One hidden irrep whose grad_out rows do not fit shared memory beside two
    edge stages (256x6e against L = 6 edges: 21 paths, 51,456 floats per atom)
    is refused with CGTP_ERR_SIZE, not planned into an invalid kernel."""
    with pytest.raises(C.CgtpError) as e:
        C.Plan("33x1o+17x4o+256x6e", "1x0e+1x1o+1x2e+1x3o+1x4e+1x5o+1x6e",
               "339x1o+340x2o+612x2e+596x3e+613x4o+885x4e+885x5o+852x6o+1091x6e", 6)
    assert e.value.status == 6 and "shared memory" in str(e.value)


def _defines(src):
    return {m.group(1): int(m.group(2)) for m in re.finditer(r"^#define (\w+) (-?\d+)\s*$", src, re.M)}


def _check_copies(src):
    """Every row copy the generated kernel makes into shared memory: the
    source range inside its global row (W: NU, x: DIN, grad_out: DOUT), the
    destination inside its staging slot (WS, XS, GS per edge), and every bulk
    (TMA) copy on 16-byte boundaries with a multiple of 16 bytes.  Returns
    (copies checked, problems)."""
    d = _defines(src)
    DIN, DOUT, NU = d["DIN"], d["DOUT"], d["NU"]
    WS, XS, GS = d.get("WS", 0), d.get("XS", 0), d.get("GS", 0)
    bad, n = [], 0
    for m in re.finditer(r"t < (\d+); t \+= 32\) sg\[(\d+) \+ t\] = grow\[(\d+) \+ t\]", src):
        N, D, S = map(int, m.groups())
        n += 1
        if not (S + N <= DOUT and D + N <= GS):
            bad.append(m.group(0))
    recognised = 0
    for arr, row, width, slot in (("sW", "WROW", NU, WS), ("sX", "XROW", DIN, XS),
                                  ("sWt", "WTROW", NU, WS), ("sXt", "XTROW", DIN, XS)):
        for m in re.finditer(r"t < nb \* (\d+); t \+= 32\) \{ const int b = t / \d+, q = t - b \* \d+; " + arr
                             + r"\[b \* (\d+) \+ (\d+) \+ q\] = " + row + r"\(b\)\[(\d+) \+ q\]", src):
            N, stride, D, S = map(int, m.groups())
            n += 1
            if not (S + N <= width and D + N <= stride == slot):
                bad.append(m.group(0))
        for m in re.finditer(r"bulk_g2s(?:_stream)?\(smem_u32\(" + arr + r" \+ b \* (\d+) \+ (\d+)\), " + row
                             + r"\(b\) \+ (\d+), (\d+),", src):
            stride, D, S, B = map(int, m.groups())
            n += 1
            recognised += 1
            if not (B % 16 == 0 and S % 4 == 0 and D % 4 == 0 and width % 4 == 0 and stride % 4 == 0
                    and S + B // 4 <= width and D + B // 4 <= stride == slot):
                bad.append(m.group(0))
    for m in re.finditer(r"bulk_g2s(?:_stream)?\(smem_u32\(sg \+ (\d+)\), grow \+ (\d+), (\d+),", src):
        D, S, B = map(int, m.groups())
        n += 1
        recognised += 1
        if not (B % 16 == 0 and S % 4 == 0 and D % 4 == 0 and DOUT % 4 == 0
                and S + B // 4 <= DOUT and D + B // 4 <= GS):
            bad.append(m.group(0))
    # one copy for a chunk's consecutive W rows (only W rows are contiguous)
    for m in re.finditer(r"bulk_g2s_stream\(smem_u32\((sWt?|sXt?)\), (WT?ROW|XT?ROW)\(0\), \(u32\)nb \* (\d+),", src):
        B = int(m.group(3))
        n += 1
        recognised += 1
        if not (m.group(1) in ("sW", "sWt") and m.group(2) in ("WROW", "WTROW") and B == 4 * NU and WS == NU
                and B % 16 == 0):
            bad.append(m.group(0))
    total = len(re.findall(r"\bbulk_g2s(?:_stream)?\(smem_u32", src))
    if total != recognised:
        bad.append(f"{total - recognised} bulk copies of an unrecognised form")
    # L2 prefetches of W: whole rows of the chunk, or row pieces, inside the
    # row, 16-byte aligned, multiples of 16 bytes
    pre = 0
    for m in re.finditer(r"bulk_prefetch_l2\(wrow \+ (\d+), (\d+)\)", src):
        S, B = map(int, m.groups())
        n += 1
        pre += 1
        if not (S % 4 == 0 and B % 16 == 0 and S + B // 4 <= NU):
            bad.append(m.group(0))
    for m in re.finditer(r"bulk_prefetch_l2\(W \+ \(size_t\)(?:pe|__ldg\(eid \+ pe \+ lane\)) \* NU, "
                         r"(?:\(u32\)npf \* )?(\d+)\)", src):
        n += 1
        pre += 1
        if not (int(m.group(1)) == 4 * NU and NU % 4 == 0):
            bad.append(m.group(0))
    if pre != len(re.findall(r"\bbulk_prefetch_l2\((?!const void)", src)):  # calls, not the definition
        bad.append("prefetches of an unrecognised form")
    return n, bad


def _check_layout(src, smem, backward):
    """Shared-memory layout of a generated kernel, from its defines: the
    regions of a stage (W, x, Y, C-hat, dY partials) in order without
    overlap; mbarriers and stage records below the first stage; the stage
    ring, the grad_out buffers and the store staging after one another
    within the planned dynamic shared memory; every offset a multiple of 16
    bytes (TMA destinations)."""
    d = _defines(src)
    NB, NW, NS, DE = d["NB"], d["NW"], d["NSTAGE"], d["DE"]
    mt = 2 if d.get("TAN", 0) else 1  # tangent kernels stage every piece twice
    off = [d["OFF_W"], d["OFF_X"], d["OFF_Y"], d["OFF_CH"], d["OFF_DY"]]
    size = [4 * mt * NB * d["WS"], 4 * mt * NB * d["XS"], 4 * mt * NB * DE, 4 * mt * NB * d["CHS"],
            4 * NW * NB * DE if backward else 0]
    bad = [f"region {k}" for k in range(4) if off[k] + size[k] > off[k + 1]]
    if off[4] + size[4] > d["STAGE_BYTES"]:
        bad.append("dY partials past the stage")
    if any(v % 16 for v in off + [d["STAGE_BYTES"], d["OFF_STAGE"], d["OFF_G"], d["OFF_WB"]]):
        bad.append("offset not 16-byte aligned")
    # the header below the first stage: full/empty/chat barriers (8 bytes
    # each, 8-byte aligned), the grad_out barriers, the int4 stage records and
    # the edge range (16-byte aligned), in order and without overlap
    hdr = [(0, 8 * NS, 8), (8 * NS, 8 * NS, 8), (d["OFF_CHAT"], 8 * NS, 8), (d["OFF_GFULL"], 16, 8),
           (d["OFF_GEMPTY"], 16, 8), (d["OFF_DESC"], 16 * NS, 16), (d["OFF_RANGE"], 16, 16)]
    for (o0, n0, a0), (o1, _, _) in zip(hdr, hdr[1:]):
        if o0 + n0 > o1:
            bad.append(f"header region at {o0} overlaps the next at {o1}")
    for o0, n0, a0 in hdr:
        if o0 % a0:
            bad.append(f"header region at {o0} not {a0}-byte aligned")
    if hdr[-1][0] + hdr[-1][1] > d["OFF_STAGE"]:
        bad.append("header past the first stage")
    if d["OFF_STAGE"] + NS * d["STAGE_BYTES"] > d["OFF_G"]:
        bad.append("stage ring past the grad_out buffers")
    gbytes = d.get("GBUF", 0) * 4 * d.get("GS", 0) if backward else 0
    if d["OFF_G"] + gbytes > d["OFF_WB"]:
        bad.append("grad_out buffers past the store staging")
    if not (d["OFF_WB"] + 4 * NW * d.get("WB", 0) <= smem <= 227 * 1024):
        bad.append(f"end {d['OFF_WB'] + 4 * NW * d.get('WB', 0)} vs planned {smem}")
    return bad


@pytest.mark.parametrize("irreps", [WL.CONFIGS[n] for n in NAMES] + [
    dict(irreps_in=a, irreps_edge=b, irreps_out=c) for a, b, c in ODD], ids=NAMES + [f"odd{k}" for k in range(len(ODD))])
@pytest.mark.parametrize("prefetch,tform,packed", [("0", "1", ""), ("4", "1", ""), ("0", "0", "0"), ("0", "1", "1")],
                         ids=["default", "prefetch4", "staged_chat_scalar_fwd", "packed_fwd"])
def test_generated_copies_stay_in_bounds(irreps, prefetch, tform, packed, compile_only, monkeypatch, tmp_path):
    """The generated kernels' row copies into shared memory and their L2
    prefetches, read from the generated source (checked here so that a
    mistake fails on the CPU rather than faulting a GPU), for the default
    kernels, with W prefetch, with the staged-Chat backward and the scalar
    forward, and with the packed forward on every plan."""
    monkeypatch.setenv("CGTP_DUMP_SOURCE", str(tmp_path))
    monkeypatch.setenv("CGTP_PREFETCH", prefetch)
    monkeypatch.setenv("CGTP_BWD_TFORM", tform)
    monkeypatch.setenv("CGTP_FWD_PACKED", packed)
    plan = C.Plan(irreps["irreps_in"], irreps["irreps_edge"], irreps["irreps_out"], 6)
    assert f"backward form={'cg_first' if tform == '1' else 'staged_chat'}" in plan.describe()
    smem = {k: int(v) for k, v in re.findall(r"^(forward|backward): .* smem=(\d+)", plan.describe(), re.M)}
    files = sorted(p.name for p in tmp_path.iterdir())
    assert files == ["bwd.cu", "bwd_er.cu", "fwd.cu"]
    for f in files:
        src = (tmp_path / f).read_text()
        n, bad = _check_copies(src)
        assert n > 0 and not bad, (f, bad[:3])
        bwd = f.startswith("bwd")
        bad = _check_layout(src, smem["backward" if bwd else "forward"], bwd)
        assert not bad, (f, bad)


@pytest.mark.parametrize("fwd", ["", "tangent", "sum"], ids=["planner", "tangent_fwd", "sum_fwd"])
@pytest.mark.parametrize("name", ["tiny", "lmax2", "lmax2_wide", "lmax3", "case5"])
def test_tangent_kernels_copies_and_layout(name, fwd, compile_only, monkeypatch, tmp_path):
    """The double backward's kernels (built on request): the tangent backward
    and the tangent forward (every staged piece doubled) and/or the
    accumulating forward; the same copy and layout checks.  Unless one is
    fixed, both forwards are built and the first call chooses by timing."""
    monkeypatch.setenv("CGTP_DUMP_SOURCE", str(tmp_path))
    monkeypatch.setenv("CGTP_DBWD_FWD", fwd)
    c = WL.CONFIGS[name]
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    assert plan.prepare_double_backward()
    desc = plan.describe()
    built = {"": ["cgtp_fwd_tan", "cgtp_fwd_acc"], "tangent": ["cgtp_fwd_tan"], "sum": ["cgtp_fwd_acc"]}[fwd]
    smem = {k: int(v) for k, v in re.findall(r"^(cgtp_fwd_tan|cgtp_fwd_acc|cgtp_bwd_tan) .* smem=(\d+)", desc, re.M)}
    assert set(smem) == set(built) | {"cgtp_bwd_tan"}, smem
    assert ("double backward forward=undecided" in desc) == (fwd == "")
    # every backward role has edges in the tangent backward's chunks: a role
    # takes the edges b with b % nph == ph, so the chunk must hold nph edges
    nph = max(int(v) for v in re.findall(r"^  brole \d+: .* ph=\d+/(\d+)", desc, re.M))
    nb = int(re.search(r"^#define NB (\d+)", (tmp_path / "bwd_tan.cu").read_text(), re.M).group(1))
    assert nb >= nph, (nb, nph)
    for f, kname in [(k[5:] + ".cu", k) for k in built] + [("bwd_tan.cu", "cgtp_bwd_tan")]:
        src = (tmp_path / f).read_text()
        assert ("#define TAN 1" in src) == (kname != "cgtp_fwd_acc")
        if kname == "cgtp_fwd_acc":
            body = src.split("extern \"C\"", 1)[0]
            assert "red_add(&orow[" in body and "orow[" not in body.replace("red_add(&orow[", "")
        n, bad = _check_copies(src)
        assert n > 0 and not bad, (f, bad[:3])
        bad = _check_layout(src, smem[kname], f.startswith("bwd"))
        assert not bad, (f, bad)


def test_copy_check_catches_planted_mistakes():
    head = "#define DIN 64\n#define DOUT 128\n#define NU 96\n#define WS 96\n#define XS 64\n#define GS 128\n"
    ok = head + ("bulk_g2s(smem_u32(sW + b * 96 + 0), WROW(b) + 32, 256, bar);\n"
                 "for (int t = lane; t < 16; t += 32) sg[0 + t] = grow[100 + t];\n")
    assert _check_copies(ok) == (2, [])
    planted = [
        "bulk_g2s(smem_u32(sW + b * 96 + 0), WROW(b) + 33, 256, bar);\n",   # source off 16 bytes
        "bulk_g2s(smem_u32(sW + b * 96 + 0), WROW(b) + 32, 260, bar);\n",   # size not 16-byte multiple
        "bulk_g2s(smem_u32(sW + b * 96 + 64), WROW(b) + 32, 256, bar);\n",  # past the W slot
        "for (int t = lane; t < 16; t += 32) sg[0 + t] = grow[120 + t];\n",  # past the grad_out row
        "if (lane == 0) bulk_g2s_stream(smem_u32(sX), XROW(0), (u32)nb * 256, bar, pol);\n",  # gathered rows
        "bulk_g2s(smem_u32(sY + 4), yrow, 64, bar);\n",                      # unknown form
    ]
    for p in planted:
        n, bad = _check_copies(head + p)
        assert bad, p


def test_layout_check_catches_a_misaligned_header():
    """A three-stage header whose stage records would start off a 16-byte
    boundary (int4 stores) fails the layout check."""
    good = ("#define NB 2\n#define NW 5\n#define NSTAGE 3\n#define DE 16\n#define WS 64\n#define XS 64\n"
            "#define CHS 64\n#define OFF_W 0\n#define OFF_X 512\n#define OFF_Y 1024\n#define OFF_CH 1152\n"
            "#define OFF_DY 1664\n#define STAGE_BYTES 1664\n#define OFF_STAGE 512\n#define OFF_G 5504\n"
            "#define OFF_WB 5504\n#define OFF_CHAT 48\n#define OFF_GFULL 80\n#define OFF_GEMPTY 96\n"
            "#define OFF_DESC 112\n#define OFF_RANGE 160\n")
    assert not _check_layout(good, 5504, False)
    bad = good.replace("#define OFF_GFULL 80\n#define OFF_GEMPTY 96\n#define OFF_DESC 112\n#define OFF_RANGE 160",
                       "#define OFF_GFULL 72\n#define OFF_GEMPTY 88\n#define OFF_DESC 104\n#define OFF_RANGE 152")
    assert any("16-byte aligned" in b for b in _check_layout(bad, 5504, False))


def test_layout_check_catches_planted_mistakes():
    # W 1024 B, x 512, Y 144, C-hat 256, dY partials 576 per stage; two stages
    good = {"NB": 4, "NW": 4, "NSTAGE": 2, "DE": 9, "WS": 64, "XS": 32, "CHS": 16, "OFF_W": 0, "OFF_X": 1024,
            "OFF_Y": 1536, "OFF_CH": 1792, "OFF_DY": 2048, "STAGE_BYTES": 2688, "OFF_STAGE": 256,
            "OFF_G": 5632, "GS": 128, "GBUF": 2, "OFF_WB": 6656, "WB": 32,
            "OFF_CHAT": 32, "OFF_GFULL": 48, "OFF_GEMPTY": 64, "OFF_DESC": 80, "OFF_RANGE": 112}
    text = lambda d: "".join(f"#define {k} {v}\n" for k, v in d.items())
    assert _check_layout(text(good), 7168, True) == []
    for key, val, smem in (("OFF_X", 768, 7168),      # W region overlaps x
                           ("OFF_Y", 1544, 7168),     # not 16-byte aligned
                           ("OFF_G", 5120, 7168),     # stage ring overlaps grad_out
                           ("OFF_WB", 6400, 7168),    # grad_out buffers overlap staging
                           ("OFF_STAGE", 64, 7168),   # barriers overlap stage 0
                           ("WB", 64, 7168)):         # past the planned size
        d = dict(good)
        d[key] = val
        assert _check_layout(text(d), smem, True), key
