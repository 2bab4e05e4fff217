"""B200-native recurrent KDA decode (placeholder; binding added with the C-ABI)."""
