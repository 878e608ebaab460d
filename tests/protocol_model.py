"""Random-schedule executor for models of the kernels' mbarrier protocols (test helper, no tests).

A model is a set of roles, each a generator of operations in program order, and a table of
barriers with their arrival counts.  Operations:
    ("wait", bar, k[, kind])         parity wait for the completion of phase k of `bar`; the
                                     role receives True, or False when the wait timed out; kind
                                     "drain" marks the waits of a role's exit path, "sync" a
                                     named barrier (bar.sync), which has no timeout
    ("arrive", bar, k)               one arrival, meant for phase k
    ("read", key, tag)               synchronous read of a buffer, expecting version `tag`
    ("write", key, tag)              synchronous write of version `tag`
    ("rmw", key, tag_in, tag_out)    read then write
    ("peek", key)                    the role receives the buffer's current version (a flag)
    ("tma", keys, tag, bar, k)       asynchronous copy writing version `tag` into every buffer in
                                     `keys`; on landing it arrives on `bar` for phase k
    ("mma", reads, writes)           asynchronous tensor-core work of this role: reads and writes
                                     lists of (key, tag), in flight until its commit completes
    ("commit", bar, k)               the role's MMAs since its last commit complete as one group
                                     and then arrive on `bar` for phase k
Freedoms of the schedule: any runnable role steps next; copies land in any order; MMA groups of
different roles complete in any order (one role's groups in issue order).  Each schedule draws a
speed for every role and a latency weight for every copy and MMA group (heavy-tailed: a few stay
in flight for a long time), so rare orders such as one copy landing many steps after later ones
are reached as well as the common ones.
Checks (ProtocolError on the first violation):
  - a parity wait is exact: when evaluated, phase k has completed or is the current one, and the
    barrier does not complete phase k + 1 while a waiter of phase k has not passed;
  - an arrival lands in the phase it is meant for;
  - a buffer is read in the expected version and not under an in-flight write; it is not written
    (synchronously, by a copy or by another role's MMA) while another access is in flight;
  - nothing deadlocks and every role finishes;
  - when the last role finishes (the block's final cluster barrier, then the release of tensor
    memory), no copy and no MMA group is still in flight.
With timeouts=True the schedule may also let any blocked wait run out (a drain wait, marked
"drain", only with drain_timeouts=True).  From the first timeout on, the barriers behave as the
hardware's do (a parity wait passes when the completed-phase count has the other parity; arrivals
just count) and the buffer checks stop, since a timed-out kernel's outputs are void; what must
still hold is the exit check: every role that gave up has waited for its own copies and MMAs.
"""
import random


class ProtocolError(AssertionError):
    pass


class Model:
    def __init__(self, barriers, roles, seed, timeouts=False, drain_timeouts=False, init=None):
        self.rng = random.Random(seed)
        self.timeouts, self.drain_timeouts = timeouts, drain_timeouts
        self.failed = False  # a wait has timed out
        self.bars = {b: {"count": c, "arr": 0, "n": 0} for b, c in barriers.items()}
        self.res = {}
        for key, tag in (init or {}).items():  # state set up before the roles start
            self.r(key)["tag"] = tag
        self.agents = {name: {"gen": gen, "op": None, "done": False, "wait": None,
                              "speed": self.rng.choice((1.0, 1.0, 0.3, 0.05))}
                       for name, gen in roles.items()}
        self.tma = []
        self.open = {name: [] for name in roles}
        self.queue = {name: [] for name in roles}
        self.gid = 0

    def fail(self, what):
        raise ProtocolError(what)

    def r(self, key):
        return self.res.setdefault(key, {"tag": None, "reads": [], "writes": []})

    # ---- barriers
    def arrive(self, bar, phase, who):
        b = self.bars[bar]
        if phase != b["n"] and not self.failed:
            self.fail(f"{who}: arrival for phase {phase} on {bar} in phase {b['n']}")
        b["arr"] += 1
        if b["arr"] == b["count"]:
            b["arr"] = 0
            b["n"] += 1
            m = b["n"] - 1
            for name, a in self.agents.items():
                if self.failed:
                    break
                if a["wait"] and a["wait"][0] == bar and a["wait"][1] < m:
                    self.fail(f"{name}: {bar} completed phase {m} while it still waited for "
                              f"phase {a['wait'][1]}")

    def passable(self, bar, k, who):
        n = self.bars[bar]["n"]
        if self.failed:
            return (n & 1) != (k & 1)
        if n < k:
            self.fail(f"{who}: waits for phase {k} of {bar}, which has completed only {n}")
        if n >= k + 2:
            self.fail(f"{who}: waits for phase {k} of {bar}, which has completed {n}")
        return n == k + 1

    # ---- buffers
    def sync_read(self, key, tag, who):
        r = self.r(key)
        if self.failed:
            return
        if r["writes"]:
            self.fail(f"{who}: reads {key} while an asynchronous write is in flight")
        if r["tag"] != tag:
            self.fail(f"{who}: reads {key} as {tag}, finds {r['tag']}")

    def sync_write(self, key, tag, who):
        r = self.r(key)
        if self.failed:
            r["tag"] = tag
            return
        if r["reads"] or r["writes"]:
            self.fail(f"{who}: writes {key} while an asynchronous access is in flight")
        r["tag"] = tag

    def issue_mma(self, who, reads, writes):
        gid = self.gid
        self.gid += 1
        for key, tag in ([] if self.failed else reads):
            r = self.r(key)
            mine = [w for w in r["writes"] if w[0] == who]
            if any(w[0] != who for w in r["writes"]):
                self.fail(f"{who}: MMA reads {key} while another write is in flight")
            have = mine[-1][2] if mine else r["tag"]
            if have != tag:
                self.fail(f"{who}: MMA reads {key} as {tag}, finds {have}")
        for key, _ in ([] if self.failed else writes):
            r = self.r(key)
            if any(x[0] != who for x in r["reads"]) or any(x[0] != who for x in r["writes"]):
                self.fail(f"{who}: MMA writes {key} while another access is in flight")
        for key, _ in reads:
            self.r(key)["reads"].append((who, gid))
        for key, tag in writes:
            self.r(key)["writes"].append((who, gid, tag))
        self.open[who].append(gid)

    def latency(self):
        return self.rng.choice((1.0, 1.0, 1.0, 0.2, 0.02, 0.002))

    def complete_group(self, who):
        g = self.queue[who].pop(0)
        ids = set(g["ids"])
        for r in self.res.values():
            for w in r["writes"]:
                if w[0] == who and w[1] in ids:
                    r["tag"] = w[2]
            r["writes"] = [w for w in r["writes"] if not (w[0] == who and w[1] in ids)]
            r["reads"] = [x for x in r["reads"] if not (x[0] == who and x[1] in ids)]
        self.arrive(g["bar"], g["phase"], who)

    def issue_tma(self, keys, tag, bar, phase, who):
        cid = ("copy", self.gid)
        self.gid += 1
        for key in keys:
            r = self.r(key)
            if (r["reads"] or r["writes"]) and not self.failed:
                self.fail(f"{who}: copy of {tag} into {key} under an asynchronous access")
            r["writes"].append((cid, None, tag))
        self.tma.append((cid, keys, tag, bar, phase, self.latency()))

    def complete_tma(self, idx):
        cid, keys, tag, bar, phase, _ = self.tma.pop(idx)
        for key in keys:
            r = self.r(key)
            r["writes"] = [w for w in r["writes"] if w[0] != cid]
            r["tag"] = tag
        self.arrive(bar, phase, "copy")

    # ---- roles
    def runnable(self, name):
        a = self.agents[name]
        if a["done"]:
            return False
        if a["op"] is not None and a["op"][0] == "wait":
            return self.passable(a["op"][1], a["op"][2], name)
        return True

    def step(self, name):
        a = self.agents[name]
        if a["op"] is None:
            try:
                a["op"] = a["gen"].send(a.pop("send", None))
            except StopIteration:
                a["done"] = True
                if all(x["done"] for x in self.agents.values()) and (
                        self.tma or any(self.queue.values()) or any(self.open.values())):
                    self.fail("the block leaves with copies or MMAs in flight")
                return
            if a["op"][0] == "wait":
                a["wait"] = (a["op"][1], a["op"][2])
                self.passable(a["op"][1], a["op"][2], name)
            return
        op, a["op"] = a["op"], None
        kind = op[0]
        if kind == "wait":
            a["wait"] = None
            a["send"] = True
        elif kind == "arrive":
            self.arrive(op[1], op[2], name)
        elif kind == "read":
            self.sync_read(op[1], op[2], name)
        elif kind == "write":
            self.sync_write(op[1], op[2], name)
        elif kind == "peek":
            a["send"] = self.r(op[1])["tag"]
        elif kind == "rmw":
            self.sync_read(op[1], op[2], name)
            self.sync_write(op[1], op[3], name)
        elif kind == "tma":
            self.issue_tma(op[1], op[2], op[3], op[4], name)
        elif kind == "mma":
            self.issue_mma(name, op[1], op[2])
        elif kind == "commit":
            self.queue[name].append({"ids": self.open[name], "bar": op[1], "phase": op[2],
                                     "w": self.latency()})
            self.open[name] = []
        else:
            raise ValueError(kind)

    def run(self, max_steps=500000):
        for _ in range(max_steps):
            cands = [("role", n) for n in self.agents if self.runnable(n)]
            cands += [("tma", i) for i in range(len(self.tma))]
            cands += [("mma", w) for w in self.queue if self.queue[w]]
            if self.timeouts:
                for n, a in self.agents.items():
                    op = a["op"]
                    if (not a["done"] and op is not None and op[0] == "wait" and
                            (len(op) < 4 or (op[3] == "drain" and self.drain_timeouts)) and
                            not self.passable(op[1], op[2], n)):
                        cands.append(("timeout", n))
            weights = [0.02 if k == "timeout" else
                       self.agents[x]["speed"] if k == "role" else
                       self.tma[x][5] if k == "tma" else self.queue[x][0]["w"] for k, x in cands]
            if not cands:
                left = [n for n, a in self.agents.items() if not a["done"]]
                if left:
                    self.fail(f"deadlock: {[(n, self.agents[n]['op']) for n in left]}")
                return
            kind, x = self.rng.choices(cands, weights)[0]
            if kind == "timeout":
                self.failed = True
                a = self.agents[x]
                a["op"], a["wait"], a["send"] = None, None, False
            elif kind == "role":
                self.step(x)
            elif kind == "tma":
                self.complete_tma(x)
            else:
                self.complete_group(x)
        raise AssertionError("schedule did not finish")


def count_caught(make, seeds):
    """How many of the seeds' schedules raise a ProtocolError."""
    caught = 0
    for seed in seeds:
        try:
            make(seed).run()
        except ProtocolError:
            caught += 1
    return caught
