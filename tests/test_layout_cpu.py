"""Host logic of the workspace layouts (csrc/layout.cuh), compiled as plain
C++ with g++: every region aligned, inside the workspace, disjoint from every
other region, the grouped-prefill region after the decode one, and the sizes
the library reports (k3moe_workspace_size) covering them."""
import json
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mxfp4_routed_expert_softmax_b200", "csrc")

DRIVER = r'''
#include <cstdio>
#include <cstdlib>
#include "layout.cuh"
using namespace k3;
int main(int argc, char **argv) {
    const int d = atoi(argv[1]), ff = atoi(argv[2]), E = atoi(argv[3]), k = atoi(argv[4]), ffs = atoi(argv[5]);
    const int Tp = atoi(argv[6]);
    const Layout L = make_layout(d, ff, E, k, ffs);
    printf("{\"decode\": {");
    const size_t dv[] = {L.hdr, L.logits, L.idx, L.wt, L.uniq_blob, L.uniq_eid, L.uniq_mask, L.uniq_slot, L.part,
                         L.cnt, L.xn, L.tmap, L.tcache, L.xb, L.xsf, L.hb, L.hsf, L.xbf, L.hsb, L.spart, L.icnt,
                         L.total};
    const char *dn[] = {"hdr", "logits", "idx", "wt", "uniq_blob", "uniq_eid", "uniq_mask", "uniq_slot", "part",
                        "cnt", "xn", "tmap", "tcache", "xb", "xsf", "hb", "hsf", "xbf", "hsb", "spart", "icnt", "total"};
    for (int i = 0; i < 22; ++i) printf("%s\"%s\": %zu", i ? ", " : "", dn[i], dv[i]);
    printf(", \"router_part_len\": %d", router_part_len(d));
    printf("}");
    if (Tp > 0) {
        const PLayout P = make_playout(L.total, d, ff, E, k, ffs, Tp);
        const size_t pv[] = {P.lg, P.idx, P.wt, P.hist, P.ecnt, P.eoff, P.goff, P.perm, P.pw, P.grp, P.itg, P.itd,
                             P.ploc, P.xg, P.xgs, P.xbf, P.hb, P.hsf, P.hsb, P.o, P.xn, P.total};
        const char *pn[] = {"lg", "idx", "wt", "hist", "ecnt", "eoff", "goff", "perm", "pw", "grp", "itg", "itd",
                            "ploc", "xg", "xgs", "xbf", "hb", "hsf", "hsb", "o", "xn", "total"};
        printf(", \"prefill\": {");
        for (int i = 0; i < 22; ++i) printf("%s\"%s\": %zu", i ? ", " : "", pn[i], pv[i]);
        printf(", \"ngr\": %d, \"ngs\": %d}", P.ngr, P.ngs);
    }
    printf("}\n");
    return 0;
}
'''


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    d = tmp_path_factory.mktemp("layout")
    src = d / "layout_driver.cpp"
    src.write_text(DRIVER)
    exe = d / "layout_driver"
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-D__host__=", "-D__device__=", "-I", CSRC, str(src), "-o",
                           str(exe)])
    return str(exe)


def layout(driver, shape, Tp):
    out = subprocess.check_output([driver, *map(str, shape), str(Tp)], text=True)
    return json.loads(out)


SHAPES = [(7168, 1536, 896, 16, 1536), (256, 128, 32, 4, 128), (512, 256, 64, 8, 192), (256, 192, 64, 32, 0),
          (512, 512, 128, 6, 64)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("Tp", [0, 9, 512, 8192])
def test_regions_are_aligned_ordered_and_disjoint(driver, shape, Tp):
    lay = layout(driver, shape, Tp)
    dec = dict(lay["decode"])
    ls = dec.pop("router_part_len")
    starts = [v for k, v in dec.items() if k != "total"]
    assert starts == sorted(starts) and len(set(starts)) == len(starts)
    assert all(v % 256 == 0 for v in dec.values())
    assert dec["hdr"] == 0 and starts[-1] < dec["total"]
    if Tp:
        pf = lay["prefill"]
        ps = [v for k, v in pf.items() if k not in ("total", "ngr", "ngs")]
        assert ps[0] >= dec["total"], "the prefill region overlaps the decode layout"
        assert ps == sorted(ps) and all(v % 256 == 0 for v in ps)
        assert ps[-1] < pf["total"]
        d, ff, E, k, ffs = shape
        # the outputs per (token, slot) come last and take T*(k+1)*d fp32
        assert pf["total"] - pf["o"] >= Tp * (k + 1) * d * 4
        # a group per 32 pairs, plus one partial group per expert at most
        assert pf["ngr"] >= Tp * k // 32 and pf["ngs"] == (-(-Tp // 32) if ffs else 0)


@pytest.mark.parametrize("shape", SHAPES)
def test_decode_regions_hold_their_contents(driver, shape):
    """The regions whose size depends on the shape: the router's part sums
    [2][E][d/Ls][4] fp32 (Ls = 512 where d allows it), the normalised input
    [8][d] bf16, and 8 tensor maps per expert plus 4 for the shared expert."""
    d, ff, E, k, ffs = shape
    dec = dict(layout(driver, shape, 0)["decode"])
    ls = dec.pop("router_part_len")
    assert ls in (512, 256, 128, 64) and d % ls == 0
    assert ls == max(x for x in (512, 256, 128, 64) if d % x == 0)
    names = [n for n in dec if n != "total"] + ["total"]
    size = {n: dec[names[i + 1]] - dec[n] for i, n in enumerate(names[:-1])}
    assert size["part"] >= 2 * E * (d // ls) * 4 * 4
    assert size["cnt"] >= 2 * E * 4
    assert size["xn"] >= 8 * d * 2
    assert size["tmap"] >= (E * 8 + 4) * 128


@pytest.mark.parametrize("shape", SHAPES)
def test_library_sizes_cover_the_layouts(driver, shape):
    import mxfp4_routed_expert_softmax_b200 as m
    dims = m.make_dims(*shape)
    dec = layout(driver, shape, 0)["decode"]["total"]
    assert m.k3moe_workspace_size(dims, 8) == dec
    for T in (9, 512, 8192):
        assert m.k3moe_workspace_size(dims, T) == layout(driver, shape, T)["prefill"]["total"]
