"""B200-native fused selective scan (S6): Python binding of libmambascan."""
