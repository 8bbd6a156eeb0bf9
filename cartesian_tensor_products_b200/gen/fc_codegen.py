"""Emit the generated CUDA headers of libflashcart from the exact algebra.

Product-side generator: run as a script (the build does) to (re)write
cartesian_tensor_products_b200/csrc/generated/*.cuh.  It uses only
fc_algebra (exact rationals) and never the test reference.

What is generated (FlashCart, arXiv 2610.06409):
  * path tables: admissible (l1,l2)->l3 ordered by l3, l1, l2; P_l per
    output rank; the App. D output offsets off(l) = sum_{l'<l}(2l'+1)P_l';
  * direction tensors T_l(u) (App. B) as straight-line polynomials in u;
  * per-edge matrices M_eta[a][b1] = sum_b2 K_eta[a][b1][b2] y_b2, where K
    are the bilinear coefficients of Sec. 3 and y = T(r-hat) (Sec. 4 Eq. 1
    shares y_e across channels, so M_eta is formed once per edge);
  * for the receiver-sorted forward (Alg. 1), the output rows are cut into
    warp groups; each group gets straight-line code that forms its M
    entries, loads its x rows and w paths, and accumulates
    z_{u eta k a} += w_{e eta k} sum_b M[a,b] x_{v k b}.
"""
import os
import sys
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import fc_algebra as A  # noqa: E402

OUTDIR = os.path.join(os.path.dirname(HERE), "csrc", "generated")


def flit(x):
    """float literal of an exact rational"""
    v = float(x)
    if v == int(v) and abs(v) < 1e6:
        return "%d.0f" % int(v)
    return "%.9ef" % v


# ---------------------------------------------------------------------------
# tables
# ---------------------------------------------------------------------------

class Tables:
    def __init__(self, L):
        self.L = L
        self.paths = A.paths(L, L, L)
        self.P = len(self.paths)
        self.Pl = [sum(1 for p in self.paths if p[2] == l) for l in range(L + 1)]
        self.eta = []
        seen = [0] * (L + 1)
        for p in self.paths:
            self.eta.append(seen[p[2]])
            seen[p[2]] += 1
        self.zoff = []
        o = 0
        for l in range(L + 1):
            self.zoff.append(o)
            o += (2 * l + 1) * self.Pl[l]
        self.zrow = o
        self.K = [A.path_coefficients(*p) for p in self.paths]
        self.ypoly = {l: A.direction_polys(l) for l in range(L + 1)}

    def zslot(self, p, a, sum_paths=False):
        l3 = self.paths[p][2]
        if sum_paths:
            return l3 * l3 + a
        return self.zoff[l3] + a * self.Pl[l3] + self.eta[p]

    def mrow(self, p, a):
        """nonzero (b1, {b2: coef}) of row a of M_p"""
        l1, l2, l3 = self.paths[p]
        out = []
        for b1 in range(2 * l1 + 1):
            terms = {b2: self.K[p][a][b1][b2] for b2 in range(2 * l2 + 1)
                     if self.K[p][a][b1][b2] != 0}
            if terms:
                out.append((b1, terms))
        return out

    def is_identity(self, p):
        l1, l2, l3 = self.paths[p]
        if l2 != 0 or l1 != l3:
            return False
        n = 2 * l1 + 1
        return all(self.K[p][a][b][0] == (1 if a == b else 0)
                   for a in range(n) for b in range(n))

    def row_cost(self, p, a):
        if self.is_identity(p):
            return 1
        return sum(1 for _ in self.mrow(p, a))


# ---------------------------------------------------------------------------
# partition of output rows into warp groups (forward kernel)
# ---------------------------------------------------------------------------

def partition_rows(T, G):
    """Rows (p, a) in order of l1 (descending), then path, then a; cut into
    G contiguous groups of near-equal cost."""
    order = sorted(range(T.P), key=lambda p: (-T.paths[p][0], p))
    rows = [(p, a) for p in order for a in range(2 * T.paths[p][2] + 1)]
    cost = [T.row_cost(p, a) + 0.25 for (p, a) in rows]
    remaining = sum(cost)
    groups, cur, acc = [], [], 0.0
    target = remaining / G
    for i, r in enumerate(rows):
        if cur and acc + cost[i] / 2 > target and len(groups) < G - 1:
            groups.append(cur)
            remaining -= acc
            target = remaining / (G - len(groups))
            cur, acc = [], 0.0
        cur.append(r)
        acc += cost[i]
    groups.append(cur)
    while len(groups) < G:
        groups.append([])
    return groups


# ---------------------------------------------------------------------------
# emission helpers
# ---------------------------------------------------------------------------

def mono_expr(m, names=("ux", "uy", "uz")):
    f = []
    for k, e in enumerate(m):
        f += [names[k]] * e
    return "*".join(f) if f else "1.0f"


def poly_expr(poly):
    terms = []
    for m, c in sorted(poly.items()):
        terms.append("(%s)*%s" % (flit(c), mono_expr(m)))
    return " + ".join(terms) if terms else "0.0f"


def lincomb_expr(terms, var):
    """sum coef * var(b) with exact coefficients"""
    out = []
    for b, c in sorted(terms.items()):
        if c == 1:
            out.append(var(b))
        elif c == -1:
            out.append("-" + var(b))
        else:
            out.append("%s*%s" % (flit(c), var(b)))
    return " + ".join(out).replace("+ -", "- ")


class GroupCode:
    """Straight-line code of one warp group of the forward kernel."""

    def __init__(self, T, rows, gid):
        self.T, self.rows, self.gid = T, rows, gid
        self.paths = []                       # global path ids, in order
        for p, a in rows:
            if p not in self.paths:
                self.paths.append(p)
        self.prow = {p: [a for (q, a) in rows if q == p] for p in self.paths}
        # x rows (component index within node row) needed
        xr = []
        for p in self.paths:
            l1 = T.paths[p][0]
            for a in self.prow[p]:
                if T.is_identity(p):
                    b_used = [a]
                else:
                    b_used = [b1 for b1, _ in T.mrow(p, a)]
                for b in b_used:
                    if l1 * l1 + b not in xr:
                        xr.append(l1 * l1 + b)
        self.xrows = sorted(xr)
        # M entries (non-identity rows)
        self.ment = []                        # (p, a, b1, {b2: coef})
        for p in self.paths:
            if T.is_identity(p):
                continue
            for a in self.prow[p]:
                for b1, terms in T.mrow(p, a):
                    self.ment.append((p, a, b1, terms))
        self.NM = len(self.ment)
        self.NMP = (self.NM + 3) // 4 * 4     # padded to float4
        s = self.NMP // 4
        if s % 2 == 0:
            s += 1                            # odd float4 stride: conflict-free
        self.MSTRIDE = max(4, 4 * s)
        self.NA = len(rows)

    def y_needed(self):
        need = set()
        for (p, a, b1, terms) in self.ment:
            l2 = self.T.paths[p][1]
            for b2 in terms:
                need.add((l2, b2))
        return sorted(need)

    def emit(self, L):
        T = self.T
        g = self.gid
        o = []
        o.append("template <> struct FwdGroup<%d, %d, %d> {" % (L, NGROUPS[L], g))
        o.append("  static constexpr int NA = %d;   // output rows (float4 accumulators)" % self.NA)
        o.append("  static constexpr int NX = %d;   // x rows loaded per edge" % len(self.xrows))
        o.append("  static constexpr int NWP = %d;  // weight paths loaded per edge" % len(self.paths))
        o.append("  static constexpr int NM = %d;   // M entries per edge" % self.NM)
        o.append("  static constexpr int MSTRIDE = %d;  // floats per edge row in smem" % self.MSTRIDE)
        # ---- make_m
        o.append("  static __device__ __forceinline__ void make_m(float ux, float uy, float uz, float* __restrict__ mrow) {")
        if self.NM:
            for (l2, b2) in self.y_needed():
                if l2 == 0:
                    o.append("    const float y_%d_%d = 1.0f;" % (l2, b2))
                else:
                    o.append("    const float y_%d_%d = %s;" % (l2, b2, poly_expr(T.ypoly[l2][b2])))
            vals = []
            for (p, a, b1, terms) in self.ment:
                l2 = T.paths[p][1]
                vals.append(lincomb_expr(terms, lambda b, l2=l2: "y_%d_%d" % (l2, b)))
            while len(vals) % 4:
                vals.append("0.0f")
            for q in range(len(vals) // 4):
                o.append("    st_f4(mrow + %d, %s, %s, %s, %s);" % (4 * q, *vals[4 * q:4 * q + 4]))
        else:
            o.append("    (void)ux; (void)uy; (void)uz; (void)mrow;")
        o.append("  }")
        # ---- loads
        o.append("  static __device__ __forceinline__ void load_x(const float* __restrict__ xv, int C, float4 (&xr)[NX]) {")
        for i, r in enumerate(self.xrows):
            o.append("    xr[%d] = ld_x4(xv + %d * C);" % (i, r))
        o.append("  }")
        o.append("  static __device__ __forceinline__ void load_w(const float* __restrict__ we, int C, float4 (&wr)[NWP]) {")
        for i, p in enumerate(self.paths):
            o.append("    wr[%d] = ld_w4(we + %d * C);" % (i, p))
        o.append("  }")
        # ---- accumulate
        o.append("  static __device__ __forceinline__ void accum(float4 (&acc)[NA], const float4 (&xr)[NX], const float4 (&wr)[NWP], const float* __restrict__ m) {")
        if self.NM:
            for q in range(self.NMP // 4):
                o.append("    const float4 mq%d = ld_s4(m + %d);" % (q, 4 * q))
        mi = 0
        ai = 0
        acc_of = {}
        for (p, a) in self.rows:
            acc_of[(p, a)] = ai
            ai += 1
        xidx = {r: i for i, r in enumerate(self.xrows)}
        comp = "xyzw"
        for pi, p in enumerate(self.paths):
            l1, l2, l3 = T.paths[p]
            o.append("    // path (%d,%d)->%d rows %s" % (l1, l2, l3, self.prow[p]))
            if T.is_identity(p):
                for a in self.prow[p]:
                    o.append("    acc[%d] = fma4(wr[%d], xr[%d], acc[%d]);" % (acc_of[(p, a)], pi, xidx[l1 * l1 + a], acc_of[(p, a)]))
                continue
            rows_p = self.prow[p]
            # entries of this path in M order
            ents = [(a, b1) for (pp, a, b1, _) in self.ment if pp == p]
            base = mi
            mi += len(ents)
            bset = sorted(set(b for _, b in ents))
            input_side = len(bset) <= len(rows_p)
            if input_side:
                for b in bset:
                    o.append("    const float4 t%d_%d = mul4(wr[%d], xr[%d]);" % (pi, b, pi, xidx[l1 * l1 + b]))
                for k, (a, b) in enumerate(ents):
                    q, c = divmod(base + k, 4)
                    o.append("    acc[%d] = fma4s(mq%d.%s, t%d_%d, acc[%d]);" % (acc_of[(p, a)], q, comp[c], pi, b, acc_of[(p, a)]))
            else:
                for a in rows_p:
                    first = True
                    for k, (aa, b) in enumerate(ents):
                        if aa != a:
                            continue
                        q, c = divmod(base + k, 4)
                        if first:
                            o.append("    float4 s%d_%d = mul4s(mq%d.%s, xr[%d]);" % (pi, a, q, comp[c], xidx[l1 * l1 + b]))
                            first = False
                        else:
                            o.append("    s%d_%d = fma4s(mq%d.%s, xr[%d], s%d_%d);" % (pi, a, q, comp[c], xidx[l1 * l1 + b], pi, a))
                    o.append("    acc[%d] = fma4(wr[%d], s%d_%d, acc[%d]);" % (acc_of[(p, a)], pi, pi, a, acc_of[(p, a)]))
        o.append("  }")
        # ---- store
        o.append("  static __device__ __forceinline__ void store(float* __restrict__ zu, int C, int sum_paths, const float4 (&acc)[NA]) {")
        o.append("    if (!sum_paths) {")
        for (p, a) in self.rows:
            o.append("      st_z4(zu + %d * C, acc[%d]);" % (T.zslot(p, a), acc_of[(p, a)]))
        o.append("    } else {")
        for (p, a) in self.rows:
            o.append("      red_add4(zu + %d * C, acc[%d]);" % (T.zslot(p, a, True), acc_of[(p, a)]))
        o.append("    }")
        o.append("  }")
        o.append("};")
        return "\n".join(o)


NGROUPS = {2: 4, 3: 8, 4: 16}


def emit_fwd(L, G):
    T = Tables(L)
    groups = partition_rows(T, G)
    codes = [GroupCode(T, rows, g) for g, rows in enumerate(groups)]
    out = []
    out.append("// Generated by gen/fc_codegen.py -- do not edit.")
    out.append("// Receiver-sorted forward, rank %d: %d paths, %d output rows, %d warp groups." % (L, T.P, T.zrow, G))
    for c in codes:
        cost = sum(T.row_cost(p, a) for p, a in c.rows)
        out.append("//   group %d: %d rows, %d M entries, %d x rows, %d w paths, cost %d" %
                   (c.gid, c.NA, c.NM, len(c.xrows), len(c.paths), cost))
    out.append("#pragma once")
    out.append('#include "../fc_device.cuh"')
    out.append("namespace fc {")
    out.append("template <> struct FwdMeta<%d> {" % L)
    out.append("  static constexpr int G = %d;           // warp groups = warps per CTA" % G)
    out.append("  static constexpr int MAXSTRIDE = %d;   // largest per-edge M row (floats)" % max(c.MSTRIDE for c in codes))
    out.append("  static constexpr int P = %d;           // paths" % T.P)
    out.append("  static constexpr int ZROW = %d;        // output components per channel" % T.zrow)
    out.append("};")
    for c in codes:
        out.append(c.emit(L))
    out.append("}  // namespace fc")
    return "\n".join(out) + "\n", T, codes


def emit_tables(Ls):
    out = ["// Generated by gen/fc_codegen.py -- do not edit.",
           "// Path tables (FlashCart Sec. 2 admissible paths; App. D layout).",
           "#pragma once", "namespace fc {"]
    for L in Ls:
        T = Tables(L)
        out.append("// rank %d: paths ordered by l3, then l1, then l2" % L)
        out.append("constexpr int kNumPaths%d = %d;" % (L, T.P))
        out.append("constexpr int kZRow%d = %d;  // output components per channel (paths separate)" % (L, T.zrow))
        out.append("constexpr int kPathL1_%d[] = {%s};" % (L, ", ".join(str(p[0]) for p in T.paths)))
        out.append("constexpr int kPathL2_%d[] = {%s};" % (L, ", ".join(str(p[1]) for p in T.paths)))
        out.append("constexpr int kPathL3_%d[] = {%s};" % (L, ", ".join(str(p[2]) for p in T.paths)))
    out.append("}  // namespace fc")
    return "\n".join(out) + "\n"


def main():
    os.makedirs(OUTDIR, exist_ok=True)
    written = []
    for L in (2, 3, 4):
        src, _, _ = emit_fwd(L, NGROUPS[L])
        path = os.path.join(OUTDIR, "fc_fwd_L%d.cuh" % L)
        with open(path, "w") as f:
            f.write(src)
        written.append(path)
    path = os.path.join(OUTDIR, "fc_tables.cuh")
    with open(path, "w") as f:
        f.write(emit_tables((2, 3, 4)))
    written.append(path)
    return written


if __name__ == "__main__":
    for p in main():
        print(p)
