"""B200-native selective scan (Mamba S6): forward, backward and decode step."""
