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



def write_if_changed(path, src):
    """Write src to path unless the file already holds it (keeps the mtime,
    so the incremental build recompiles only what a change touches)."""
    if os.path.exists(path):
        with open(path) as f:
            if f.read() == src:
                return
    with open(path, "w") as f:
        f.write(src)


def flit(x):
    """float literal of an exact rational"""
    v = float(x)
    if v == int(v) and abs(v) < 1e6:
        return "%d.0f" % int(v)
    return "%.9ef" % v


# ---------------------------------------------------------------------------
# tables
# ---------------------------------------------------------------------------

# Odd-J (Levi-Civita) path sets are emitted under template key L + ODD_KEY.
ODD_KEY = 16


class Tables:
    def __init__(self, L, odd=False):
        self.L = L
        self.odd = odd
        self.paths = A.odd_paths(L, L, L) if odd else A.paths(L, L, L)
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
        coeffs = A.odd_path_coefficients if odd else A.path_coefficients
        self.K = [coeffs(*p) for p in self.paths]
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

def partition_rows(T, G, row_weight=0.0):
    """Rows (p, a) in order of l1 (descending), then path, then a; cut into
    G contiguous groups of near-equal cost (per-lane FMAs of the row plus
    row_weight per accumulator)."""
    order = sorted(range(T.P), key=lambda p: (-T.paths[p][0], p))
    rows = [(p, a) for p in order for a in range(2 * T.paths[p][2] + 1)]
    cost = [T.row_cost(p, a) + 0.25 + row_weight for (p, a) in rows]
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


def ycomp(l, c):
    """index of component c of rank l in the stacked direction tensor"""
    return l * l + c


class GroupCode:
    """Straight-line code of one warp group of the forward kernel.

    A lane owns 4 channels (one float4).  Per edge the group needs the x
    rows its M entries touch and the weight rows of its paths; both are
    staged in a per-warp shared-memory ring, each lane copying and reading
    only its own 16-byte slice.  M entries are formed in registers from the
    direction tensor y of the edge (same value in every lane) and used for
    the 4 channels of the lane."""

    def __init__(self, T, rows, gid):
        self.T, self.rows, self.gid = T, rows, gid
        self.paths = []                       # global path ids, in order
        for p, a in rows:
            if p not in self.paths:
                self.paths.append(p)
        self.prow = {p: [a for (q, a) in rows if q == p] for p in self.paths}
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
        self.ment = []                        # (p, a, b1, {b2: coef}) in use order
        self.form = {}                        # path -> True: input side (t_b = w x_b)
        for p in self.paths:
            if T.is_identity(p):
                continue
            ents = [(a, b1, terms) for a in self.prow[p] for b1, terms in T.mrow(p, a)]
            bset = sorted(set(b for _, b, _ in ents))
            self.form[p] = len(bset) <= len(self.prow[p])
            if self.form[p]:
                # b-major: consecutive FMAs update different accumulators
                ents.sort(key=lambda e: (e[1], e[0]))
            else:
                # term-major over the rows of the path
                per_row = {a: [e for e in ents if e[0] == a] for a in self.prow[p]}
                ents = []
                depth = max(len(v) for v in per_row.values())
                for j in range(depth):
                    for a in self.prow[p]:
                        if j < len(per_row[a]):
                            ents.append(per_row[a][j])
            for (a, b1, terms) in ents:
                self.ment.append((p, a, b1, terms))
        self.NM = len(self.ment)
        self.NA = len(rows)
        self.NROW = len(self.xrows) + len(self.paths)
        # entries equal up to sign share one stored value
        self.uniq, self.usign, ukey = [], [], {}
        for (p, a, b1, terms) in self.ment:
            l2 = T.paths[p][1]
            t = tuple(sorted(terms.items()))
            neg = tuple((b, -c) for b, c in t)
            key = (l2, min(t, neg))
            sign = 1 if key[1] == t else -1
            if key not in ukey:
                ukey[key] = len(self.uniq)
                self.uniq.append((l2, dict(key[1])))
            self.usign.append((ukey[key], sign))
        # identity paths (l2 = 0) use the stored edge scale s when an
        # envelope is on
        self.sidx = None
        if any(T.is_identity(p) for p in self.paths):
            key = (0, ((0, 1),))
            if key not in ukey:
                ukey[key] = len(self.uniq)
                self.uniq.append((0, {0: 1}))
            self.sidx = ukey[key]
        self.NU = len(self.uniq)
        q = max(1, (self.NU + 3) // 4)
        if q % 2 == 0:
            q += 1                            # odd float4 stride: conflict-free stores
        self.MSTRIDE = 4 * q

    def y_needed(self):
        need = set()
        for (p, a, b1, terms) in self.ment:
            l2 = self.T.paths[p][1]
            for b2 in terms:
                need.add((l2, b2))
        for (l2, terms) in self.uniq:
            for b2 in terms:
                need.add((l2, b2))
        return sorted(need)

    def emit(self, L, G):
        T = self.T
        g = self.gid
        comp = "xyzw"
        o = []
        o.append("template <> struct FwdGroup<%d, %d, %d> {" % (L, G, g))
        o.append("  static constexpr int NA = %d;    // output rows (float4 accumulators)" % self.NA)
        o.append("  static constexpr int NX = %d;    // x rows staged per edge" % len(self.xrows))
        o.append("  static constexpr int NWP = %d;   // weight rows staged per edge" % len(self.paths))
        o.append("  static constexpr int NROW = %d;  // staged 512-byte rows per edge" % self.NROW)
        o.append("  static constexpr int NM = %d;    // M entries per edge (%d distinct up to sign)" % (self.NM, self.NU))
        o.append("  static constexpr int MSTRIDE = %d;  // floats per edge row of the M window" % self.MSTRIDE)
        o.append("  static constexpr int RING_OFF = %d;  // staging ring (floats into shared memory)" % self.ring_off)
        o.append("  static constexpr int MWIN_OFF = %d;  // M window (floats into shared memory)" % self.mwin_off)
        # ---- M entries of one edge (lane-per-edge), from the unit direction
        o.append("  template <bool ENV>")
        o.append("  static __device__ __forceinline__ void make_m(float ux, float uy, float uz, float s, float* __restrict__ mrow) {")
        if self.NM or self.sidx is not None:
            for (l2, b2) in self.y_needed():
                if l2 == 0:
                    o.append("    const float y_%d_%d = 1.0f;" % (l2, b2))
                else:
                    o.append("    const float y_%d_%d = %s;" % (l2, b2, poly_expr(T.ypoly[l2][b2])))
            for env in (True, False):
                vals = []
                for k, (l2, terms) in enumerate(self.uniq):
                    e = lincomb_expr(terms, lambda b, l2=l2: "y_%d_%d" % (l2, b))
                    if not env and k == self.sidx:
                        e = "0.0f"          # the scale slot is read only under an envelope
                    vals.append(("s*(%s)" % e) if env else e)
                while len(vals) % 4:
                    vals.append("0.0f")
                o.append("    if constexpr (%sENV) {" % ("" if env else "!"))
                for q in range(len(vals) // 4):
                    o.append("      st_f4(mrow + %d, %s, %s, %s, %s);" % (4 * q, *vals[4 * q:4 * q + 4]))
                o.append("    }")
        else:
            o.append("    (void)ux; (void)uy; (void)uz; (void)s; (void)mrow;")
        o.append("  }")
        # ---- issue the copies of one edge
        o.append("  static __device__ __forceinline__ void issue(float* st, const float* __restrict__ xv, const float* __restrict__ we, int C, bool xok, bool ok) {")
        for i, r in enumerate(self.xrows):
            o.append("    cp_async16(st + %d, xv + %d * C, xok);" % (128 * i, r))
        for i, p in enumerate(self.paths):
            o.append("    cp_async16(st + %d, we + %d * C, ok);" % (128 * (len(self.xrows) + i), p))
        o.append("  }")
        # ---- accumulate one edge
        o.append("  // ENV: an edge envelope scales every M entry; the identity paths")
        o.append("  // (l2 = 0) then read the stored scale instead of using w x directly")
        o.append("  template <bool ENV>")
        o.append("  static __device__ __forceinline__ void accum(float4 (&acc)[NA], const float* st, const float* __restrict__ m) {")
        for i, r in enumerate(self.xrows):
            o.append("    const float4 x%d = ld_s4(st + %d);" % (r, 128 * i))
        for i, p in enumerate(self.paths):
            o.append("    const float4 w%d = ld_s4(st + %d);" % (i, 128 * (len(self.xrows) + i)))
        acc_of = {r: i for i, r in enumerate(self.rows)}
        loaded = set()
        mi = 0
        for pi, p in enumerate(self.paths):
            l1, l2, l3 = T.paths[p]
            o.append("    // path (%d,%d)->%d rows %s" % (l1, l2, l3, self.prow[p]))
            if T.is_identity(p):
                q, c = divmod(self.sidx, 4)
                o.append("    if constexpr (ENV) {")
                o.append("      const float sc = m[%d];" % self.sidx)
                for a in self.prow[p]:
                    i = acc_of[(p, a)]
                    o.append("      acc[%d] = fma4s(sc, mul4(w%d, x%d), acc[%d]);" % (i, pi, l1 * l1 + a, i))
                o.append("    } else {")
                for a in self.prow[p]:
                    i = acc_of[(p, a)]
                    o.append("      acc[%d] = fma4(w%d, x%d, acc[%d]);" % (i, pi, l1 * l1 + a, i))
                o.append("    }")
                continue
            rows_p = self.prow[p]
            ents = [(a, b1) for (pp, a, b1, _) in self.ment if pp == p]
            names = []
            for k in range(len(ents)):
                ui, sign = self.usign[mi + k]
                q, c = divmod(ui, 4)
                if q not in loaded:
                    o.append("    const float4 mq%d = ld_s4(m + %d);" % (q, 4 * q))
                    loaded.add(q)
                names.append(("" if sign > 0 else "-") + "mq%d.%s" % (q, comp[c]))
            mi += len(ents)
            if self.form[p]:
                bset = sorted(set(b for _, b in ents))
                for b in bset:
                    o.append("    const float4 t%d_%d = mul4(w%d, x%d);" % (pi, b, pi, l1 * l1 + b))
                for k, (a, b) in enumerate(ents):
                    i = acc_of[(p, a)]
                    o.append("    acc[%d] = fma4s(%s, t%d_%d, acc[%d]);" % (i, names[k], pi, b, i))
            else:
                started = set()
                for k, (a, b) in enumerate(ents):
                    if a not in started:
                        o.append("    float4 s%d_%d = mul4s(%s, x%d);" % (pi, a, names[k], l1 * l1 + b))
                        started.add(a)
                    else:
                        o.append("    s%d_%d = fma4s(%s, x%d, s%d_%d);" % (pi, a, names[k], l1 * l1 + b, pi, a))
                for a in rows_p:
                    i = acc_of[(p, a)]
                    o.append("    acc[%d] = fma4(w%d, s%d_%d, acc[%d]);" % (i, pi, pi, a, i))
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


def emit_direction(L):
    """T_l(u) for l <= L, stacked: y[l*l + c]"""
    o = ["template <> struct Direction<%d> {" % L,
         "  static constexpr int NY = %d;" % ((L + 1) ** 2),
         "  static __device__ __forceinline__ void eval(float ux, float uy, float uz, float (&y)[NY]) {"]
    T = Tables(L)
    for l in range(L + 1):
        for c in range(2 * l + 1):
            o.append("    y[%d] = %s;" % (ycomp(l, c), poly_expr(T.ypoly[l][c]) if l else "1.0f"))
    o.append("  }")
    o.append("};")
    return "\n".join(o)


NGROUPS = {1: 2, 2: 4, 3: 4, 4: 8, 5: 24}
ROW_WEIGHT = {1: 0.0, 2: 0.0, 3: 0.0, 4: 4.0, 5: 4.0}
STAGES = {1: 3, 2: 3, 3: 3, 4: 2, 5: 2}
MWIN = 16
FWD_WARPS = 2


def emit_fwd(L, G, odd=False):
    T = Tables(L, odd)
    key = L + ODD_KEY if odd else L
    groups = partition_rows(T, G, ROW_WEIGHT[L])
    codes = [GroupCode(T, rows, g) for g, rows in enumerate(groups)]
    out = []
    out.append("// Generated by gen/fc_codegen.py -- do not edit.")
    out.append("// Receiver-sorted forward, rank %d%s: %d paths, %d output rows, %d warp groups." %
               (L, " odd-J paths (template key %d)" % key if odd else "", T.P, T.zrow, G))
    for c in codes:
        cost = sum(T.row_cost(p, a) for p, a in c.rows)
        out.append("//   group %d: %d rows, %d M entries, %d x rows, %d w rows, %d FMA/channel" %
                   (c.gid, c.NA, c.NM, len(c.xrows), len(c.paths), cost))
    out.append("#pragma once")
    out.append('#include "../fc_device.cuh"')
    out.append("namespace fc {")
    out.append("template <> struct FwdMeta<%d> {" % key)
    out.append("  static constexpr int G = %d;           // warp groups = warps per CTA" % G)
    out.append("  static constexpr int S = %d;           // staging ring depth (edges)" % STAGES[L])
    out.append("  static constexpr int MAXROW = %d;      // largest staged rows per edge of a group" % max(c.NROW for c in codes))
    out.append("  static constexpr int P = %d;           // paths" % T.P)
    out.append("  static constexpr int ZROW = %d;        // output components per channel" % T.zrow)
    if G <= 4:
        # one CTA = the G groups of one receiver (one warp per SMSP)
        off = 0
        for c in codes:
            c.ring_off = off
            off += STAGES[L] * 128 * c.NROW
        for c in codes:
            c.mwin_off = off
            off += MWIN * c.MSTRIDE
        warp_floats, warps, total = 0, G, off
    else:
        # one CTA = one group for FWD_WARPS receivers (group-major blocks)
        nrow = max(c.NROW for c in codes)
        mstride = max(c.MSTRIDE for c in codes)
        for c in codes:
            c.ring_off = 0
            c.mwin_off = STAGES[L] * 128 * nrow
        warp_floats = STAGES[L] * 128 * nrow + MWIN * mstride
        warps, total = FWD_WARPS, FWD_WARPS * warp_floats
    out.append("  static constexpr int MWIN = %d;        // edges per M window" % MWIN)
    out.append("  static constexpr bool GROUP_MAJOR = %s;" % ("true" if G > 4 else "false"))
    out.append("  static constexpr int WARPS = %d;       // warps per CTA" % warps)
    out.append("  static constexpr int WARP_FLOATS = %d; // shared memory of one warp (group-major)" % warp_floats)
    out.append("  static constexpr int SMEM_FLOATS = %d; // shared memory of a CTA" % total)
    out.append("};")
    for c in codes:
        out.append(c.emit(key, G))
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
    for L in (1, 2, 3, 4, 5):
        src, _, _ = emit_fwd(L, NGROUPS[L])
        path = os.path.join(OUTDIR, "fc_fwd_L%d.cuh" % L)
        write_if_changed(path, src)
        written.append(path)
    path = os.path.join(OUTDIR, "fc_tables.cuh")
    write_if_changed(path, emit_tables((1, 2, 3, 4, 5)))
    written.append(path)
    return written



# ---------------------------------------------------------------------------
# receiver-sorted VJP (App. C Eq. C1 summed as in Algorithm 2)
# ---------------------------------------------------------------------------

def direction_derivative_polys(l):
    """d T_l(u)_c / d u_j as polynomials (j = x, y, z), for every component."""
    out = []
    for poly in A.direction_polys(l):
        out.append([A.p_diff(poly, j) for j in range(3)])
    return out


def partition_paths(T, G, cost):
    """Whole paths (h = M^T g needs all rows of a path) in order of l1
    (descending), cut into G contiguous groups of near-equal cost."""
    order = sorted(range(T.P), key=lambda p: (-T.paths[p][0], p))
    c = [cost(p) for p in order]
    remaining = sum(c)
    groups, cur, acc = [], [], 0.0
    target = remaining / G
    for i, p in enumerate(order):
        if cur and acc + c[i] / 2 > target and len(groups) < G - 1:
            groups.append(cur)
            remaining -= acc
            target = remaining / (G - len(groups))
            cur, acc = [], 0.0
        cur.append(p)
        acc += c[i]
    groups.append(cur)
    while len(groups) < G:
        groups.append([])
    return groups


def vjp_path_cost(T, p):
    l1, l2, l3 = T.paths[p]
    nm = sum(len(T.mrow(p, a)) for a in range(2 * l3 + 1)) if not T.is_identity(p) else 2 * l1 + 1
    nk = sum(1 for a in range(2 * l3 + 1) for b1 in range(2 * l1 + 1)
             for b2 in range(2 * l2 + 1) if T.K[p][a][b1][b2] != 0)
    return 2 * nm + 4 * (2 * l1 + 1) + 2 * (2 * l1 + 1) + 3 * nm + nk


class VjpGroupCode:
    """Straight-line code of one warp group of the VJP kernel (whole paths)."""

    def __init__(self, T, paths, gid):
        self.T, self.gpaths, self.gid = T, paths, gid
        L = T.L
        self.rows = [(p, a) for p in paths for a in range(2 * T.paths[p][2] + 1)]
        self.NA = len(self.rows)
        xr = []
        for p in paths:
            l1 = T.paths[p][0]
            for b in range(2 * l1 + 1):
                if l1 * l1 + b not in xr:
                    xr.append(l1 * l1 + b)
        self.xrows = sorted(xr)
        # M entries (row-major per path) and the (a, b1) -> {b2: K} terms
        self.ment = []
        for p in paths:
            l1, l2, l3 = T.paths[p]
            for a in range(2 * l3 + 1):
                for b1, terms in T.mrow(p, a):
                    self.ment.append((p, a, b1, terms))
        self.NM = len(self.ment)
        # every direction component the group touches, T_0 = 1 included: it has
        # no angular derivative, but under a radial envelope s(|r|) T_0 does
        ycomps = sorted(set((T.paths[p][1], b2) for p in paths
                            for b2 in range(2 * T.paths[p][1] + 1)))
        self.ycomps = ycomps                 # direction components with a gradient
        self.NYD = len(ycomps)
        self.NROW = len(self.xrows) + len(paths)
        self.dbase = (self.NM + 3) // 4 * 4  # offset of d y / d u in a window row
        self.ybase = self.dbase + 3 * self.NYD   # offset of s'(|r|) y
        n = self.ybase + self.NYD
        q = max(1, (n + 3) // 4)
        if q % 2 == 0:
            q += 1
        self.MSTRIDE = 4 * q

    def emit(self, L, G):
        T = self.T
        g = self.gid
        o = []
        o.append("template <> struct VjpGroup<%d, %d, %d> {" % (L, G, g))
        o.append("  static constexpr int NA = %d;    // g rows held in registers (float4)" % self.NA)
        o.append("  static constexpr int NX = %d;    // x rows staged per edge (= x_bar rows)" % len(self.xrows))
        o.append("  static constexpr int NWP = %d;   // weight rows staged per edge" % len(self.gpaths))
        o.append("  static constexpr int NROW = %d;  // staged 512-byte rows per edge" % self.NROW)
        o.append("  static constexpr int NM = %d;    // M entries per edge" % self.NM)
        o.append("  static constexpr int NYD = %d;   // direction components with a gradient" % self.NYD)
        o.append("  static constexpr int MSTRIDE = %d;  // floats per edge row of the window" % self.MSTRIDE)
        o.append("  static constexpr int RING_OFF = %d;" % self.ring_off)
        o.append("  static constexpr int MWIN_OFF = %d;" % self.mwin_off)
        # ---- window row: M pairs, then d y / d u (3 per component)
        o.append("  static __device__ __forceinline__ void make_row(float ux, float uy, float uz, float s, float sp, float* __restrict__ mrow) {")
        yneed = set(self.ycomps)
        for (p, a, b1, terms) in self.ment:
            for b2 in terms:
                yneed.add((T.paths[p][1], b2))
        for (l2, b2) in sorted(yneed):
            o.append("    const float y_%d_%d = %s;" % (l2, b2, poly_expr(T.ypoly[l2][b2]) if l2 else "1.0f"))
        vals = []
        for k, (p, a, b1, terms) in enumerate(self.ment):
            l2 = T.paths[p][1]
            vals.append("s*(%s)" % lincomb_expr(terms, lambda b, l2=l2: "y_%d_%d" % (l2, b)))
        while len(vals) < self.dbase:
            vals.append("0.0f")
        for (l2, b2) in self.ycomps:
            for j in range(3):
                vals.append("s*(%s)" % poly_expr(direction_derivative_polys(l2)[b2][j]))
        for (l2, b2) in self.ycomps:
            vals.append("sp*y_%d_%d" % (l2, b2))
        while len(vals) % 4:
            vals.append("0.0f")
        for q in range(len(vals) // 4):
            o.append("    st_f4(mrow + %d, %s, %s, %s, %s);" % (4 * q, *vals[4 * q:4 * q + 4]))
        o.append("  }")
        # ---- staging
        o.append("  static __device__ __forceinline__ void issue(float* st, const float* __restrict__ xv, const float* __restrict__ we, int C, bool xok, bool ok) {")
        for i, r in enumerate(self.xrows):
            o.append("    cp_async16(st + %d, xv + %d * C, xok);" % (128 * i, r))
        for i, p in enumerate(self.gpaths):
            o.append("    cp_async16(st + %d, we + %d * C, ok);" % (128 * (len(self.xrows) + i), p))
        o.append("  }")
        # ---- load g rows of the receiver
        o.append("  static __device__ __forceinline__ void load_g(const float* __restrict__ gu, int C, int sum_paths, float4 (&gr)[NA]) {")
        o.append("    if (!sum_paths) {")
        for i, (p, a) in enumerate(self.rows):
            o.append("      gr[%d] = ld_x4(gu + %d * C);" % (i, T.zslot(p, a)))
        o.append("    } else {")
        for i, (p, a) in enumerate(self.rows):
            o.append("      gr[%d] = ld_x4(gu + %d * C);" % (i, T.zslot(p, a, True)))
        o.append("    }")
        o.append("  }")
        # ---- one edge
        xidx = {r: i for i, r in enumerate(self.xrows)}
        gi = {r: i for i, r in enumerate(self.rows)}
        o.append("  static __device__ __forceinline__ void edge(const float4 (&gr)[NA], const float* st, const float* __restrict__ m,")
        o.append("      float4 (&xb)[NX], float (&yb)[%d], float* __restrict__ wbar_e, int C, bool act) {" % max(1, self.NYD))
        for i, r in enumerate(self.xrows):
            o.append("    const float4 x%d = ld_s4(st + %d);" % (r, 128 * i))
        ycidx = {c: i for i, c in enumerate(self.ycomps)}
        mi = 0
        loaded = set()
        for pi, p in enumerate(self.gpaths):
            l1, l2, l3 = T.paths[p]
            ents = [(a, b1, terms) for (pp, a, b1, terms) in self.ment if pp == p]
            bset = sorted(set(b for _, b, _ in ents))
            names = []
            for k in range(len(ents)):
                q, c = divmod(mi + k, 4)
                if q not in loaded:
                    o.append("    const float4 mq%d = ld_s4(m + %d);" % (q, 4 * q))
                    loaded.add(q)
                names.append("mq%d.%s" % (q, "xyzw"[c]))
            mi += len(ents)
            o.append("    { // path (%d,%d)->%d" % (l1, l2, l3))
            o.append("      const float4 w = ld_s4(st + %d);" % (128 * (len(self.xrows) + pi)))
            # h_b1 = sum_a M[a][b1] g_a  (row-major order keeps the chains apart)
            started = set()
            for k, (a, b, _) in enumerate(ents):
                ga = "gr[%d]" % gi[(p, a)]
                if b not in started:
                    o.append("      float4 h%d = mul4s(%s, %s);" % (b, names[k], ga))
                    started.add(b)
                else:
                    o.append("      h%d = fma4s(%s, %s, h%d);" % (b, names[k], ga, b))
            # w_bar = <h, x>;  x_bar += w h
            first = True
            for b in bset:
                xr = "x%d" % (l1 * l1 + b)
                if first:
                    o.append("      float4 wb = mul4(h%d, %s);" % (b, xr))
                    first = False
                else:
                    o.append("      wb = fma4(h%d, %s, wb);" % (b, xr))
                o.append("      xb[%d] = fma4(w, h%d, xb[%d]);" % (xidx[l1 * l1 + b], b, xidx[l1 * l1 + b]))
            o.append("      if (act) st_z4(wbar_e + %d * C, wb);" % p)
            # y_bar: d_(a,b1) = <g_a, w x_b1> over the lane's 4 channels, then K
            if True:
                for b in bset:
                    o.append("      const float4 t%d = mul4(w, x%d);" % (b, l1 * l1 + b))
                for k, (a, b, terms) in enumerate(ents):
                    o.append("      { const float d = dot4(gr[%d], t%d);" % (gi[(p, a)], b))
                    for b2, c in sorted(terms.items()):
                        o.append("        yb[%d] = fmaf(%s, d, yb[%d]);" % (ycidx[(l2, b2)], flit(c), ycidx[(l2, b2)]))
                    o.append("      }")
            o.append("    }")
        o.append("  }")
        # ---- u_bar = (d y / d u)^T y_bar  (uniform d y / d u from the window)
        o.append("  static __device__ __forceinline__ void ubar(const float (&yb)[%d], const float* __restrict__ m, float& ux, float& uy, float& uz, float& rho) {" % max(1, self.NYD))
        o.append("    ux = 0.0f; uy = 0.0f; uz = 0.0f; rho = 0.0f;")
        for i in range(self.NYD):
            base = self.dbase + 3 * i
            o.append("    ux = fmaf(yb[%d], m[%d], ux); uy = fmaf(yb[%d], m[%d], uy); uz = fmaf(yb[%d], m[%d], uz);" %
                     (i, base, i, base + 1, i, base + 2))
            o.append("    rho = fmaf(yb[%d], m[%d], rho);" % (i, self.ybase + i))
        o.append("  }")
        # ---- x_bar rows
        o.append("  static __device__ __forceinline__ void flush_xbar(float* __restrict__ xbv, int C, float4 (&xb)[NX]) {")
        for i, r in enumerate(self.xrows):
            o.append("    red_add4(xbv + %d * C, xb[%d]); xb[%d] = zero4();" % (r, i, i))
        o.append("  }")
        o.append("};")
        return "\n".join(o)


VJP_NGROUPS = {1: 2, 2: 4, 3: 8, 4: 8, 5: 24}
VJP_STAGES = {1: 3, 2: 3, 3: 3, 4: 2, 5: 2}
VJP_MWIN = {1: 16, 2: 16, 3: 16, 4: 8, 5: 8}
VJP_MINB = {1: 2, 2: 2, 3: 2, 4: 2, 5: 2}     # resident CTAs per SM the launch bound asks for


def emit_vjp(L, G, odd=False):
    T = Tables(L, odd)
    key = L + ODD_KEY if odd else L
    groups = partition_paths(T, G, lambda p: vjp_path_cost(T, p))
    codes = [VjpGroupCode(T, ps, g) for g, ps in enumerate(groups)]
    # every warp of a CTA runs the same group (one instruction stream per
    # SMSP), so all groups share one per-warp layout: ring, then M window
    nrow = max(c.NROW for c in codes)
    mstride = max(c.MSTRIDE for c in codes)
    for c in codes:
        c.ring_off = 0
        c.mwin_off = VJP_STAGES[L] * 128 * nrow
    off = VJP_STAGES[L] * 128 * nrow + VJP_MWIN[L] * mstride
    out = ["// Generated by gen/fc_codegen.py -- do not edit.",
           "// Receiver-sorted VJP, rank %d%s: %d paths, %d warp groups (whole paths)." %
           (L, " odd-J paths (template key %d)" % key if odd else "", T.P, G)]
    for c in codes:
        out.append("//   group %d: paths %s, %d g rows, %d M entries, %d x rows, cost %d" %
                   (c.gid, [T.paths[p] for p in c.gpaths], c.NA, c.NM, len(c.xrows),
                    sum(vjp_path_cost(T, p) for p in c.gpaths)))
    out += ["#pragma once", '#include "../fc_device.cuh"', "namespace fc {",
            "template <> struct VjpMeta<%d> {" % key,
            "  static constexpr int G = %d;" % G,
            "  static constexpr int S = %d;" % VJP_STAGES[L],
            "  static constexpr int MWIN = %d;" % VJP_MWIN[L],
            "  static constexpr int P = %d;" % T.P,
            "  static constexpr int WARP_FLOATS = %d;   // shared memory of one warp" % off,
            "  static constexpr int WARPS = 4;           // receivers per CTA (same group)",
            "  static constexpr int MINB = %d;            // CTAs per SM of the launch bound" % VJP_MINB[L],
            "  static constexpr int SMEM_FLOATS = %d;" % (4 * off),
            "};"]
    for c in codes:
        out.append(c.emit(key, G))
    out.append("}  // namespace fc")
    return "\n".join(out) + "\n", T, codes


# ---------------------------------------------------------------------------
# receiver-sorted VJP-of-VJP (App. C Eq. C2, Algorithm 3)
# ---------------------------------------------------------------------------

D2_PAIRS = ((0, 0), (0, 1), (0, 2), (1, 1), (1, 2), (2, 2))


def direction_second_derivative_polys(l):
    """d^2 T_l(u)_c / d u_i d u_j for the symmetric pairs D2_PAIRS."""
    return [[A.p_diff(A.p_diff(poly, i), j) for (i, j) in D2_PAIRS]
            for poly in A.direction_polys(l)]


def vvjp_path_cost(T, p):
    l1, l2, l3 = T.paths[p]
    nm = sum(len(T.mrow(p, a)) for a in range(2 * l3 + 1))
    nk = sum(1 for a in range(2 * l3 + 1) for b1 in range(2 * l1 + 1)
             for b2 in range(2 * l2 + 1) if T.K[p][a][b1][b2] != 0)
    return 6 * nm + 8 * (2 * l1 + 1) + (4 * nk if l2 > 0 else 0)


class VvjpGroupCode:
    """Straight-line code of one warp group of the VJP-of-VJP kernel (whole
    paths).  Per edge, path and lane (4 channels), with M = M(y) and
    Mv = M(vy) the per-edge matrices of the direction tensors and of their
    derivative along the edge-vector cotangent:
      t = w vx + vw x,  s = w x
      h = M^T g,  hv = Mv^T g
      g_hat += M t + Mv s                      (= w[f(vx,y) + f(x,vy)] + vw f(x,y))
      w_hat  = <h, vx> + <hv, x>               (= <g, f(vx,y) + f(x,vy)>)
      x_hat += w hv + vw h                     (= VJP1(g, w vy + vw y))
      y_hat += K-contraction of <g, t>          (= VJP2(g, w vx + vw x))
      y_bar += K-contraction of <g, s>          (= VJP2(g, w x), for the Hessian term)."""

    def __init__(self, T, paths, gid):
        self.T, self.gpaths, self.gid = T, paths, gid
        self.rows = [(p, a) for p in paths for a in range(2 * T.paths[p][2] + 1)]
        self.NA = len(self.rows)
        self.xrows = sorted(set(T.paths[p][0] ** 2 + b for p in paths
                                for b in range(2 * T.paths[p][0] + 1)))
        self.NX = len(self.xrows)
        self.NP = len(paths)
        self.ment = [(p, a, b1, terms) for p in paths for a in range(2 * T.paths[p][2] + 1)
                     for b1, terms in T.mrow(p, a)]
        self.NM = len(self.ment)
        # direction components with an angular derivative (T_0 = 1 has none)
        self.dcomps = sorted(set((T.paths[p][1], b2) for p in paths if T.paths[p][1] > 0
                                 for b2 in range(2 * T.paths[p][1] + 1)))
        self.ND = len(self.dcomps)
        self.NROW = 2 * self.NX + 2 * self.NP
        self.dbase = (2 * self.NM + 3) // 4 * 4      # d y / d u of dcomps (3 each)
        self.d2base = self.dbase + 3 * self.ND      # d^2 y / du du (6 each)
        self.sbase = self.d2base + 6 * self.ND      # ux uy uz wx wy wz inv_r u.vr
        n = self.sbase + 8
        q = max(1, (n + 3) // 4)
        if q % 2 == 0:
            q += 1
        self.MSTRIDE = 4 * q

    def emit(self, L, G):
        T = self.T
        o = []
        o.append("template <> struct VvjpGroup<%d, %d, %d> {" % (L, G, self.gid))
        o.append("  static constexpr int NA = %d;    // g rows (and g_hat rows) in registers" % self.NA)
        o.append("  static constexpr int NX = %d;    // x rows (and vx rows) staged per edge" % self.NX)
        o.append("  static constexpr int NP = %d;    // paths (w and vw rows staged per edge)" % self.NP)
        o.append("  static constexpr int NROW = %d;  // staged 512-byte rows per edge" % self.NROW)
        o.append("  static constexpr int NM = %d;    // entries of M (and of Mv) per edge" % self.NM)
        o.append("  static constexpr int ND = %d;    // direction components with a derivative" % self.ND)
        o.append("  static constexpr int SBASE = %d; // per-edge scalars in the window row" % self.sbase)
        o.append("  static constexpr int MSTRIDE = %d;" % self.MSTRIDE)
        o.append("  static constexpr int RING_OFF = %d;" % self.ring_off)
        o.append("  static constexpr int MWIN_OFF = %d;" % self.mwin_off)
        # ---- window row
        o.append("  static __device__ __forceinline__ void make_row(float ux, float uy, float uz, float inv_r, float vrx, float vry, float vrz, float* __restrict__ mrow) {")
        yneed = set()
        for (p, a, b1, terms) in self.ment:
            for b2 in terms:
                yneed.add((T.paths[p][1], b2))
        dneed = sorted(set(self.dcomps) | set(c for c in yneed if c[0] > 0))
        for (l2, b2) in sorted(yneed):
            o.append("    const float y_%d_%d = %s;" % (l2, b2, poly_expr(T.ypoly[l2][b2]) if l2 else "1.0f"))
        for (l2, b2) in dneed:
            d = direction_derivative_polys(l2)[b2]
            for j in range(3):
                o.append("    const float d_%d_%d_%d = %s;" % (l2, b2, j, poly_expr(d[j])))
        o.append("    const float uv = ux * vrx + uy * vry + uz * vrz;")
        o.append("    const float wx = (vrx - ux * uv) * inv_r, wy = (vry - uy * uv) * inv_r, wz = (vrz - uz * uv) * inv_r;")
        for (l2, b2) in sorted(yneed):
            if l2:
                o.append("    const float vy_%d_%d = d_%d_%d_0 * wx + d_%d_%d_1 * wy + d_%d_%d_2 * wz;" %
                         (l2, b2, l2, b2, l2, b2, l2, b2))
            else:
                o.append("    const float vy_%d_%d = 0.0f;" % (l2, b2))
        vals = []
        for (p, a, b1, terms) in self.ment:
            l2 = T.paths[p][1]
            vals.append(lincomb_expr(terms, lambda b, l2=l2: "y_%d_%d" % (l2, b)))
        for (p, a, b1, terms) in self.ment:
            l2 = T.paths[p][1]
            vals.append(lincomb_expr(terms, lambda b, l2=l2: "vy_%d_%d" % (l2, b)))
        while len(vals) < self.dbase:
            vals.append("0.0f")
        for (l2, b2) in self.dcomps:
            for j in range(3):
                vals.append("d_%d_%d_%d" % (l2, b2, j))
        for (l2, b2) in self.dcomps:
            for e in direction_second_derivative_polys(l2)[b2]:
                vals.append(poly_expr(e))
        vals += ["ux", "uy", "uz", "wx", "wy", "wz", "inv_r", "uv"]
        while len(vals) % 4:
            vals.append("0.0f")
        for q in range(len(vals) // 4):
            o.append("    st_f4(mrow + %d, %s, %s, %s, %s);" % (4 * q, *vals[4 * q:4 * q + 4]))
        o.append("  }")
        # ---- staging
        o.append("  static __device__ __forceinline__ void issue(float* st, const float* __restrict__ xv, const float* __restrict__ vxv,")
        o.append("      const float* __restrict__ we, const float* __restrict__ vwe, int C, bool xok, bool vxok, bool ok, bool vwok) {")
        for i, r in enumerate(self.xrows):
            o.append("    cp_async16(st + %d, xv + %d * C, xok);" % (128 * i, r))
        for i, r in enumerate(self.xrows):
            o.append("    cp_async16(st + %d, vxv + %d * C, vxok);" % (128 * (self.NX + i), r))
        for i, p in enumerate(self.gpaths):
            o.append("    cp_async16(st + %d, we + %d * C, ok);" % (128 * (2 * self.NX + i), p))
        for i, p in enumerate(self.gpaths):
            o.append("    cp_async16(st + %d, vwe + %d * C, vwok);" % (128 * (2 * self.NX + self.NP + i), p))
        o.append("  }")
        # ---- g rows of the receiver
        o.append("  static __device__ __forceinline__ void load_g(const float* __restrict__ gu, int C, int sum_paths, float4 (&gr)[NA]) {")
        o.append("    if (!sum_paths) {")
        for i, (p, a) in enumerate(self.rows):
            o.append("      gr[%d] = ld_x4(gu + %d * C);" % (i, T.zslot(p, a)))
        o.append("    } else {")
        for i, (p, a) in enumerate(self.rows):
            o.append("      gr[%d] = ld_x4(gu + %d * C);" % (i, T.zslot(p, a, True)))
        o.append("    }")
        o.append("  }")
        # ---- g_hat rows of the receiver (added: with summed paths several
        # groups share a slot)
        o.append("  static __device__ __forceinline__ void store_ghat(float* __restrict__ gu, int C, int sum_paths, const float4 (&gh)[NA]) {")
        o.append("    if (!sum_paths) {")
        for i, (p, a) in enumerate(self.rows):
            o.append("      red_add4(gu + %d * C, gh[%d]);" % (T.zslot(p, a), i))
        o.append("    } else {")
        for i, (p, a) in enumerate(self.rows):
            o.append("      red_add4(gu + %d * C, gh[%d]);" % (T.zslot(p, a, True), i))
        o.append("    }")
        o.append("  }")
        # ---- one edge
        xidx = {r: i for i, r in enumerate(self.xrows)}
        gi = {r: i for i, r in enumerate(self.rows)}
        dix = {c: i for i, c in enumerate(self.dcomps)}
        NDm = max(1, self.ND)
        o.append("  static __device__ __forceinline__ void edge(const float4 (&gr)[NA], float4 (&gh)[NA], const float* st,")
        o.append("      const float* __restrict__ m, float4 (&xh)[NX], float (&yh)[%d], float (&yb)[%d]," % (NDm, NDm))
        o.append("      float* __restrict__ what_e, int C, bool wstore) {")
        for i, r in enumerate(self.xrows):
            o.append("    const float4 x%d = ld_s4(st + %d);" % (r, 128 * i))
            o.append("    const float4 vx%d = ld_s4(st + %d);" % (r, 128 * (self.NX + i)))
        mi = 0
        loaded = set()

        def mname(k):
            q, c = divmod(k, 4)
            return "mq%d.%s" % (q, "xyzw"[c])

        for pi, p in enumerate(self.gpaths):
            l1, l2, l3 = T.paths[p]
            ents = [(a, b1, terms) for (pp, a, b1, terms) in self.ment if pp == p]
            bset = sorted(set(b for _, b, _ in ents))
            # the path's window quads, loaded at function scope just before their
            # first use (a quad can span two paths)
            ks = list(range(mi, mi + len(ents))) + list(range(self.NM + mi, self.NM + mi + len(ents)))
            for q in sorted(set(k // 4 for k in ks)):
                if q not in loaded:
                    o.append("    const float4 mq%d = ld_s4(m + %d);" % (q, 4 * q))
                    loaded.add(q)
            o.append("    { // path (%d,%d)->%d" % (l1, l2, l3))
            names = [mname(mi + k) for k in range(len(ents))]
            vnames = [mname(self.NM + mi + k) for k in range(len(ents))]
            mi += len(ents)
            o.append("      const float4 w = ld_s4(st + %d);" % (128 * (2 * self.NX + pi)))
            o.append("      const float4 vw = ld_s4(st + %d);" % (128 * (2 * self.NX + self.NP + pi)))
            for b in bset:
                r = l1 * l1 + b
                o.append("      const float4 t%d = fma4(w, vx%d, mul4(vw, x%d));" % (b, r, r))
                o.append("      const float4 s%d = mul4(w, x%d);" % (b, r))
            started = set()
            for k, (a, b, _) in enumerate(ents):
                ga = "gr[%d]" % gi[(p, a)]
                if b not in started:
                    o.append("      float4 h%d = mul4s(%s, %s);" % (b, names[k], ga))
                    o.append("      float4 hv%d = mul4s(%s, %s);" % (b, vnames[k], ga))
                    started.add(b)
                else:
                    o.append("      h%d = fma4s(%s, %s, h%d);" % (b, names[k], ga, b))
                    o.append("      hv%d = fma4s(%s, %s, hv%d);" % (b, vnames[k], ga, b))
                o.append("      gh[%d] = fma4s(%s, t%d, fma4s(%s, s%d, gh[%d]));" %
                         (gi[(p, a)], names[k], b, vnames[k], b, gi[(p, a)]))
            first = True
            for b in bset:
                r = l1 * l1 + b
                if first:
                    o.append("      float4 wh = fma4(hv%d, x%d, mul4(h%d, vx%d));" % (b, r, b, r))
                    first = False
                else:
                    o.append("      wh = fma4(hv%d, x%d, fma4(h%d, vx%d, wh));" % (b, r, b, r))
                o.append("      xh[%d] = fma4(w, hv%d, fma4(vw, h%d, xh[%d]));" % (xidx[r], b, b, xidx[r]))
            o.append("      if (wstore) st_z4(what_e + %d * C, wh);" % p)
            if l2 > 0:
                for k, (a, b, terms) in enumerate(ents):
                    o.append("      { const float dh = dot4(gr[%d], t%d), db = dot4(gr[%d], s%d);" %
                             (gi[(p, a)], b, gi[(p, a)], b))
                    for b2, c in sorted(terms.items()):
                        i = dix[(l2, b2)]
                        o.append("        yh[%d] = fmaf(%s, dh, yh[%d]); yb[%d] = fmaf(%s, db, yb[%d]);" %
                                 (i, flit(c), i, i, flit(c), i))
                    o.append("      }")
            o.append("    }")
        o.append("  }")
        # ---- fold y_hat, y_bar into u-space: D^T y_hat (3), G = D^T y_bar (3),
        # H_u = sum y_bar D2 (6)
        o.append("  static __device__ __forceinline__ void fold(const float (&yh)[%d], const float (&yb)[%d], const float* __restrict__ m, float (&red)[12]) {" % (NDm, NDm))
        o.append("#pragma unroll")
        o.append("    for (int i = 0; i < 12; ++i) red[i] = 0.0f;")
        for i in range(self.ND):
            b1 = self.dbase + 3 * i
            b2 = self.d2base + 6 * i
            for j in range(3):
                o.append("    red[%d] = fmaf(yh[%d], m[%d], red[%d]); red[%d] = fmaf(yb[%d], m[%d], red[%d]);" %
                         (j, i, b1 + j, j, 3 + j, i, b1 + j, 3 + j))
            for j in range(6):
                o.append("    red[%d] = fmaf(yb[%d], m[%d], red[%d]);" % (6 + j, i, b2 + j, 6 + j))
        o.append("  }")
        # ---- x_hat rows
        o.append("  static __device__ __forceinline__ void flush_xhat(float* __restrict__ xhv, int C, float4 (&xh)[NX]) {")
        for i, r in enumerate(self.xrows):
            o.append("    red_add4(xhv + %d * C, xh[%d]); xh[%d] = zero4();" % (r, i, i))
        o.append("  }")
        o.append("};")
        return "\n".join(o)


VVJP_NGROUPS = {1: 2, 2: 6, 3: 16, 4: 32}
VVJP_STAGES = {1: 2, 2: 2, 3: 2, 4: 2, 5: 2}
VVJP_MWIN = {1: 8, 2: 8, 3: 8, 4: 8, 5: 8}
# Above rank 4 every path group is its own kernel launch (registers are then
# allocated per group), and a group holds at most this many g rows.
VVJP_SPLIT_MAX_ROWS = 12


def partition_paths_capped(T, cost, max_rows, target):
    """Whole paths in order of l1 (descending), cut into contiguous groups of
    about `target` cost each, no group holding more than max_rows output rows
    (a single path larger than that is a group of its own)."""
    order = sorted(range(T.P), key=lambda p: (-T.paths[p][0], p))
    groups, cur, acc, rows = [], [], 0.0, 0
    for p in order:
        r = 2 * T.paths[p][2] + 1
        c = cost(p)
        if cur and (rows + r > max_rows or acc + c / 2 > target):
            groups.append(cur)
            cur, acc, rows = [], 0.0, 0
        cur.append(p)
        acc += c
        rows += r
    if cur:
        groups.append(cur)
    return groups


def emit_vvjp(L, G):
    T = Tables(L)
    if L > 4:
        total = sum(vvjp_path_cost(T, p) for p in range(T.P))
        groups = partition_paths_capped(T, lambda p: vvjp_path_cost(T, p), VVJP_SPLIT_MAX_ROWS,
                                        total / G)
        G = len(groups)
    else:
        groups = partition_paths(T, G, lambda p: vvjp_path_cost(T, p))
    codes = [VvjpGroupCode(T, ps, g) for g, ps in enumerate(groups)]
    nrow = max(c.NROW for c in codes)
    mstride = max(c.MSTRIDE for c in codes)
    for c in codes:
        c.ring_off = 0
        c.mwin_off = VVJP_STAGES[L] * 128 * nrow
    off = VVJP_STAGES[L] * 128 * nrow + VVJP_MWIN[L] * mstride
    out = ["// Generated by gen/fc_codegen.py -- do not edit.",
           "// Receiver-sorted VJP-of-VJP, rank %d: %d paths, %d warp groups (whole paths)." % (L, T.P, G)]
    for c in codes:
        out.append("//   group %d: paths %s, %d g rows, %d M entries, %d x rows, cost %d" %
                   (c.gid, [T.paths[p] for p in c.gpaths], c.NA, c.NM, c.NX,
                    sum(vvjp_path_cost(T, p) for p in c.gpaths)))
    out += ["#pragma once", '#include "../fc_device.cuh"', "namespace fc {",
            "template <> struct VvjpMeta<%d> {" % L,
            "  static constexpr int G = %d;" % G,
            "  static constexpr bool SPLIT = %s;   // one launch per group" % ("true" if L > 4 else "false"),
            "  static constexpr int S = %d;" % VVJP_STAGES[L],
            "  static constexpr int MWIN = %d;" % VVJP_MWIN[L],
            "  static constexpr int P = %d;" % T.P,
            "  static constexpr int WARP_FLOATS = %d;   // shared memory of one warp" % off,
            "  static constexpr int WARPS = 4;           // receivers per CTA (same group)",
            "  static constexpr int SMEM_FLOATS = %d;" % (4 * off),
            "};"]
    for c in codes:
        out.append(c.emit(L, G))
    out.append("}  // namespace fc")
    return "\n".join(out) + "\n", T, codes


_main_fwd = main


# odd-J paths (ranks 1-4): 1, 4, 11, 23 paths
ODD_NGROUPS = {1: 1, 2: 2, 3: 4, 4: 4}
ODD_VJP_NGROUPS = {1: 1, 2: 2, 3: 4, 4: 8}


def main():
    written = _main_fwd()
    for L in (1, 2, 3, 4):
        src, _, _ = emit_fwd(L, ODD_NGROUPS[L], odd=True)
        path = os.path.join(OUTDIR, "fc_fwd_odd_L%d.cuh" % L)
        write_if_changed(path, src)
        written.append(path)
        src, _, _ = emit_vjp(L, ODD_VJP_NGROUPS[L], odd=True)
        path = os.path.join(OUTDIR, "fc_vjp_odd_L%d.cuh" % L)
        write_if_changed(path, src)
        written.append(path)
    for L in (1, 2, 3, 4, 5):
        src, _, _ = emit_vjp(L, VJP_NGROUPS[L])
        path = os.path.join(OUTDIR, "fc_vjp_L%d.cuh" % L)
        write_if_changed(path, src)
        written.append(path)
        src, _, _ = emit_vvjp(L, VVJP_NGROUPS.get(L, 48))
        path = os.path.join(OUTDIR, "fc_vvjp_L%d.cuh" % L)
        write_if_changed(path, src)
        written.append(path)
    return written



# ---------------------------------------------------------------------------
# node-local product ladder (Sec. 5 Eq. 2, path-reduced products, App. E)
# ---------------------------------------------------------------------------

def emit_ladder(L):
    """Channel-diagonal products of one node and one channel:
       B[l3^2 + c] = sum_{paths -> l3} w_p f_p(a[l1 block], b[l2 block])_c
    and their VJP (App. C Eq. C1 applied per path)."""
    T = Tables(L)
    NY = (L + 1) ** 2
    o = ["// Generated by gen/fc_codegen.py -- do not edit.",
         "// Node-local channel-diagonal products, rank %d, %d paths." % (L, T.P),
         "#pragma once", "namespace fc {",
         "template <> struct LadderTP<%d> {" % L,
         "  static constexpr int NY = %d;" % NY,
         "  static constexpr int P = %d;" % T.P]
    # forward
    o.append("  static __device__ __forceinline__ void fwd(const float (&a)[NY], const float (&b)[NY], const float (&w)[P], float (&B)[NY]) {")
    o.append("#pragma unroll")
    o.append("    for (int i = 0; i < NY; ++i) B[i] = 0.0f;")
    for p, (l1, l2, l3) in enumerate(T.paths):
        K = T.K[p]
        for c in range(2 * l3 + 1):
            terms = [(b1, b2, K[c][b1][b2]) for b1 in range(2 * l1 + 1)
                     for b2 in range(2 * l2 + 1) if K[c][b1][b2] != 0]
            if not terms:
                continue
            expr = " + ".join("%s*(a[%d]*b[%d])" % (flit(k), l1 * l1 + b1, l2 * l2 + b2)
                              for b1, b2, k in terms)
            o.append("    B[%d] = fmaf(w[%d], %s, B[%d]);" % (l3 * l3 + c, p, expr, l3 * l3 + c))
    o.append("  }")
    # full ladder: every path kept, written at its output slot
    # zoff[l3] + c P_l3 + eta of a [ZROW][C] row (stride C)
    o.append("  static constexpr int ZROW = %d;" % T.zrow)
    o.append("  static __device__ __forceinline__ void fwd_paths(const float (&a)[NY], const float (&b)[NY], float* __restrict__ o, int C) {")
    for p, (l1, l2, l3) in enumerate(T.paths):
        K = T.K[p]
        for c in range(2 * l3 + 1):
            terms = [(b1, b2, K[c][b1][b2]) for b1 in range(2 * l1 + 1)
                     for b2 in range(2 * l2 + 1) if K[c][b1][b2] != 0]
            expr = " + ".join("%s*(a[%d]*b[%d])" % (flit(k), l1 * l1 + b1, l2 * l2 + b2)
                              for b1, b2, k in terms) or "0.0f"
            o.append("    o[(size_t)%d * C] = %s;" % (T.zslot(p, c), expr))
    o.append("  }")
    # the same products handed to a writer: put(l3, c, eta_l3, value)
    o.append("  template <class Put>")
    o.append("  static __device__ __forceinline__ void fwd_paths_to(const float (&a)[NY], const float (&b)[NY], Put&& put) {")
    for p, (l1, l2, l3) in enumerate(T.paths):
        K = T.K[p]
        for c in range(2 * l3 + 1):
            terms = [(b1, b2, K[c][b1][b2]) for b1 in range(2 * l1 + 1)
                     for b2 in range(2 * l2 + 1) if K[c][b1][b2] != 0]
            expr = " + ".join("%s*(a[%d]*b[%d])" % (flit(k), l1 * l1 + b1, l2 * l2 + b2)
                              for b1, b2, k in terms) or "0.0f"
            o.append("    put(%d, %d, %d, %s);" % (l3, c, T.eta[p], expr))
    o.append("  }")
    # VJP: g is the gradient of B
    o.append("  static __device__ __forceinline__ void vjp(const float (&a)[NY], const float (&b)[NY], const float (&w)[P], const float (&g)[NY],")
    o.append("                                             float (&abar)[NY], float (&bbar)[NY], float (&wbar)[P]) {")
    for p, (l1, l2, l3) in enumerate(T.paths):
        K = T.K[p]
        o.append("    { // path (%d,%d)->%d" % (l1, l2, l3))
        # h_b1 = d<g, f>/da_b1 = sum K g_c b_b2; then abar += w h and, since f
        # is linear in a, w_bar = <g, f> = sum_b1 a_b1 h_b1
        hs = []
        for b1 in range(2 * l1 + 1):
            t = ["%s*(g[%d]*b[%d])" % (flit(K[c][b1][b2]), l3 * l3 + c, l2 * l2 + b2)
                 for c in range(2 * l3 + 1) for b2 in range(2 * l2 + 1) if K[c][b1][b2] != 0]
            if t:
                o.append("      const float h%d = %s;" % (b1, " + ".join(t)))
                o.append("      abar[%d] = fmaf(w[%d], h%d, abar[%d]);" % (l1 * l1 + b1, p, b1, l1 * l1 + b1))
                hs.append(b1)
        if hs:
            o.append("      wbar[%d] += %s;" % (p, " + ".join("a[%d]*h%d" % (l1 * l1 + b1, b1) for b1 in hs)))
        for b2 in range(2 * l2 + 1):
            t = ["%s*(g[%d]*a[%d])" % (flit(K[c][b1][b2]), l3 * l3 + c, l1 * l1 + b1)
                 for c in range(2 * l3 + 1) for b1 in range(2 * l1 + 1) if K[c][b1][b2] != 0]
            if t:
                o.append("      bbar[%d] = fmaf(w[%d], %s, bbar[%d]);" % (l2 * l2 + b2, p, " + ".join(t), l2 * l2 + b2))
        o.append("    }")
    o.append("  }")
    # full ladder VJP: every path has its own output gradient, get(l3, c, eta)
    o.append("  template <class Get>")
    o.append("  static __device__ __forceinline__ void vjp_paths(const float (&a)[NY], const float (&b)[NY], Get&& get,")
    o.append("                                                   float (&abar)[NY], float (&bbar)[NY]) {")
    for p, (l1, l2, l3) in enumerate(T.paths):
        K = T.K[p]
        o.append("    { // path (%d,%d)->%d" % (l1, l2, l3))
        o.append("      float g[%d];" % (2 * l3 + 1))
        for c in range(2 * l3 + 1):
            o.append("      g[%d] = get(%d, %d, %d);" % (c, l3, c, T.eta[p]))
        for b1 in range(2 * l1 + 1):
            t = ["%s*(g[%d]*b[%d])" % (flit(K[c][b1][b2]), c, l2 * l2 + b2)
                 for c in range(2 * l3 + 1) for b2 in range(2 * l2 + 1) if K[c][b1][b2] != 0]
            if t:
                o.append("      abar[%d] += %s;" % (l1 * l1 + b1, " + ".join(t)))
        for b2 in range(2 * l2 + 1):
            t = ["%s*(g[%d]*a[%d])" % (flit(K[c][b1][b2]), c, l1 * l1 + b1)
                 for c in range(2 * l3 + 1) for b1 in range(2 * l1 + 1) if K[c][b1][b2] != 0]
            if t:
                o.append("      bbar[%d] += %s;" % (l2 * l2 + b2, " + ".join(t)))
        o.append("    }")
    o.append("  }")
    o.append("};")
    o.append("}  // namespace fc")
    return "\n".join(o) + "\n"


_main_conv = main


def main():
    written = _main_conv()
    for L in (1, 2, 3, 4):
        path = os.path.join(OUTDIR, "fc_ladder_L%d.cuh" % L)
        write_if_changed(path, emit_ladder(L))
        written.append(path)
    return written


if __name__ == "__main__":
    for p in main():
        print(p)
